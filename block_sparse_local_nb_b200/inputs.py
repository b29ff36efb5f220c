"""Seeded synthetic inputs for the attention and tokenizer workloads.

This module holds no arithmetic of the method: it only draws random numbers
with fixed seeds, so the same inputs can be handed to the CUDA library and to
the CPU oracle.  Recipes (shapes, seeds, value distributions):

* ``fp32_n256``     fp32, batch 1 x heads 1 x n 256 x d 64, R = 1, full lengths,
                    Q, K, V ~ N(0, 1), seed 0.
* ``bf16_varlen``   bf16, 4 x 12 x 4096 x 64, R = 2; lengths L_b drawn first,
                    uniform on the integers 1024..4096; Q, K, V, dO ~ N(0, 1), seed 2.
* ``bf16_n131k``    bf16, 1 x 16 x 131072 x 128, R = 4, full; 0.5 * N(0, 1), seed 3.
* ``bf16_n1m``      bf16, 1 x 8 x 1048576 x 64, R = 8, full; N(0, 1), seed 4.
* ``dna_2p28``      2**28 ASCII bytes; each byte is 'N' with probability 0.01,
                    otherwise uniform over A/C/G/T; seed 5.

Tensors are drawn as fp32 standard normals in the order Q, K, V, dO from one
``torch.Generator`` (on the CPU for sizes the oracle handles, on the target
device for the large workloads), then scaled and cast to the run dtype; the
oracle is always handed the cast values.
"""

from __future__ import annotations

from dataclasses import dataclass, field

import numpy as np
import torch


@dataclass(frozen=True)
class AttnWorkload:
    name: str
    dtype: str  # "f32" or "bf16"
    batch: int
    heads: int
    n: int
    d: int
    R: int
    seed: int
    scale: float = 1.0
    varlen: tuple | None = None  # (lo, hi) inclusive range of sequence lengths
    backward: bool = True
    desc: str = field(default="", compare=False)
    causal: bool = False  # the causal band (key blocks i - R..i, keys k <= q)


WORKLOADS = {
    "fp32_n256": AttnWorkload("fp32_n256", "f32", 1, 1, 256, 64, 1, 0, backward=False,
                              desc="fwd fp32 1x1x256x64 R=1 full"),
    "bf16_varlen": AttnWorkload("bf16_varlen", "bf16", 4, 12, 4096, 64, 2, 2, varlen=(1024, 4096),
                                desc="fwd+bwd bf16 4x12x4096x64 R=2 L~U[1024,4096]"),
    "bf16_varlen_causal": AttnWorkload("bf16_varlen_causal", "bf16", 4, 12, 4096, 64, 2, 2,
                                       varlen=(1024, 4096), causal=True,
                                       desc="fwd+bwd bf16 4x12x4096x64 R=2 causal band "
                                            "L~U[1024,4096]"),
    "bf16_n131k": AttnWorkload("bf16_n131k", "bf16", 1, 16, 131072, 128, 4, 3, scale=0.5,
                               desc="fwd+bwd bf16 1x16x131072x128 R=4 full"),
    "bf16_n1m": AttnWorkload("bf16_n1m", "bf16", 1, 8, 1048576, 64, 8, 4,
                             desc="fwd then fwd+bwd bf16 1x8x1048576x64 R=8 full"),
}

DNA_BYTES = 1 << 28
DNA_SEED = 5
DNA_N_PROB = 0.01


def torch_dtype(name: str) -> torch.dtype:
    return {"f32": torch.float32, "bf16": torch.bfloat16}[name]


def make_lengths(w: AttnWorkload) -> torch.Tensor:
    """int32 [batch] sequence lengths (drawn before the tensors for varlen)."""
    if w.varlen is None:
        return torch.full((w.batch,), w.n, dtype=torch.int32)
    g = torch.Generator().manual_seed(w.seed)
    lo, hi = w.varlen
    return torch.randint(lo, hi + 1, (w.batch,), generator=g, dtype=torch.int64).to(torch.int32)


def make_attn_inputs(w: AttnWorkload, device="cpu", batch=None, heads=None, n=None, seed=None):
    """Return (q, k, v, do, lengths) for workload ``w``.

    ``batch``/``heads``/``n``/``seed`` override the workload's values (used by
    small parity cases that keep a workload's distribution).  The generator
    lives on ``device``; lengths are always drawn on the CPU.
    """
    b = w.batch if batch is None else batch
    h = w.heads if heads is None else heads
    nn = w.n if n is None else n
    s = w.seed if seed is None else seed
    shape = (b, h, nn, w.d)
    if w.varlen is not None and batch is None and n is None and seed is None:
        lengths = make_lengths(w)
    elif w.varlen is not None:  # scaled-down varlen case: L_b uniform on n/4..n
        g = torch.Generator().manual_seed(s)
        lengths = torch.randint(max(1, nn // 4), nn + 1, (b,), generator=g, dtype=torch.int64).to(torch.int32)
    else:
        lengths = torch.full((b,), nn, dtype=torch.int32)
    g = torch.Generator(device=device).manual_seed(s)
    dt = torch_dtype(w.dtype)
    out = []
    for _ in range(4):  # Q, K, V, dO in this order
        t = torch.randn(shape, generator=g, device=device, dtype=torch.float32)
        if w.scale != 1.0:
            t.mul_(w.scale)
        out.append(t.to(dt))
    return (*out, lengths)


def random_attn_inputs(batch, heads, n, d, dtype, seed, device="cpu", scale=1.0):
    """Q, K, V, dO ~ scale * N(0, 1) drawn in that order from one seeded generator."""
    g = torch.Generator(device=device).manual_seed(seed)
    dt = torch_dtype(dtype)
    return tuple((scale * torch.randn((batch, heads, n, d), generator=g, device=device)).to(dt)
                 for _ in range(4))


def make_dna(nbytes: int = DNA_BYTES, seed: int = DNA_SEED, n_prob: float = DNA_N_PROB) -> np.ndarray:
    """uint8 ASCII DNA: 'N' with probability ``n_prob``, else uniform A/C/G/T."""
    rng = np.random.default_rng(seed)
    denom = 10000
    u = rng.integers(0, denom, size=nbytes, dtype=np.uint16)
    letters = np.frombuffer(b"ACGT", dtype=np.uint8)
    out = letters[u & 3]
    out[u < int(round(n_prob * denom))] = ord("N")
    return out


# batch of DNA sequences for the model-ID tokenizer: 8192 sequences whose base
# counts are uniform in [1024, 4101] (so the padded width is 4096 windows),
# bases as in make_dna
DNA_BATCH = 8192
DNA_BATCH_BASES = (1024, 4101)
DNA_BATCH_SEED = 6


def make_dna_batch(count: int = DNA_BATCH, bases=DNA_BATCH_BASES, seed: int = DNA_BATCH_SEED):
    """(blob uint8, offsets int64 [count + 1]): the sequences concatenated."""
    rng = np.random.default_rng(seed)
    lens = rng.integers(bases[0], bases[1] + 1, size=count).astype(np.int64)
    offsets = np.zeros(count + 1, dtype=np.int64)
    np.cumsum(lens, out=offsets[1:])
    blob = make_dna(int(offsets[-1]), seed=seed + 1000)
    return blob, offsets
