"""Training-layer glue around the C ABI (argument marshalling and buffer
allocation only; every step of the computation runs in ``libnb_b200.so``).

* :func:`collate` is the page's "Dynamic Ceiling Hardware Alignment" data path
  (NucleoByte page, section 2 item 2): a batch of DNA strings becomes one
  int64 ``[batch, n_pad]`` matrix of model input IDs, ``n_pad`` the smallest
  multiple of 32 that holds the longest sequence's k-mer windows, plus the
  per-sequence window counts that the attention takes as ``lengths``.  One
  kernel (``nb_tokenize_batch``) tokenizes, offsets and pads on the device.
* :class:`BlockSparseLocalAttention` is the page's ``torch.autograd.Function``
  integration (section 4 "Tech Stack"): forward through ``nb_attn_fwd``
  (keeping the log-sum-exp), backward through ``nb_attn_bwd`` (P recomputed
  from it).  Tensors are ``[batch, heads, n, d]``; the backward needs bf16.
"""

from __future__ import annotations

from typing import Sequence

import numpy as np
import torch

from . import binding as nb

BLOCK = 32
PAD_ID = 0


def ceiling_layout(base_counts: Sequence[int], k: int = 6) -> tuple[np.ndarray, int]:
    """Offsets (int64 [batch + 1]) of the concatenated sequences and the
    dynamic ceiling n_pad (computed by the library's nb_batch_ceiling) for
    sequences of the given base counts."""
    counts = np.asarray([int(c) for c in base_counts], dtype=np.int64)
    if (counts < 0).any():
        raise ValueError("base counts must be non-negative")
    offsets = np.zeros(counts.size + 1, dtype=np.int64)
    np.cumsum(counts, out=offsets[1:])
    return offsets, nb.nb_batch_ceiling(offsets, counts.size, k)


def collate(seqs: Sequence[bytes], k: int = 6, device=None, stream=None):
    """Model input IDs and lengths of a batch of DNA byte strings, on the device.

    Returns ``(input_ids, lengths)``: int64 ``[batch, n_pad]`` with ID 0 for
    padding, raw k-mer ID + 1 for a window of A/C/G/T and 4**k + 1 for a window
    holding any other byte; int32 ``[batch]`` window counts.  Asynchronous on
    ``stream`` (default: the current stream).
    """
    device = torch.device(device if device is not None else "cuda")
    offsets, n_pad = ceiling_layout([len(s) for s in seqs], k)
    blob = b"".join(bytes(s) for s in seqs)
    host = torch.frombuffer(bytearray(blob or b"\0"), dtype=torch.uint8).pin_memory()
    host_off = torch.from_numpy(offsets).pin_memory()
    s = stream if stream is not None else torch.cuda.current_stream(device)
    with torch.cuda.stream(s):
        dev_blob = host.to(device, non_blocking=True)
        dev_off = host_off.to(device, non_blocking=True)
        ids = torch.empty((len(seqs), n_pad), dtype=torch.int64, device=device)
        lengths = torch.empty(len(seqs), dtype=torch.int32, device=device)
    nb.nb_tokenize_batch(dev_blob, dev_off, len(seqs), k, ids, lengths, n_pad, s)
    return ids, lengths


def _dtype_code(t: torch.Tensor) -> int:
    if t.dtype == torch.bfloat16:
        return nb.NB_BF16
    if t.dtype == torch.float32:
        return nb.NB_F32
    raise TypeError(f"unsupported dtype {t.dtype} (bf16 or fp32)")


class BlockSparseLocalAttention(torch.autograd.Function):
    """O = softmax(Q K^T / sqrt(d) restricted to the band |i - j| <= R of
    32-token blocks and to keys < lengths[b]) V, with its backward.  With
    ``causal`` the band is i - R <= j <= i and keys k <= q."""

    @staticmethod
    def forward(ctx, q, k, v, lengths, R: int, causal: bool = False):
        if not (q.shape == k.shape == v.shape and q.dim() == 4):
            raise ValueError("q, k, v must share one [batch, heads, n, d] shape")
        if not (q.dtype == k.dtype == v.dtype):
            raise TypeError("q, k, v must share one dtype")
        q, k, v = q.contiguous(), k.contiguous(), v.contiguous()
        batch, heads, n, d = q.shape
        if lengths is not None:
            lengths = lengths.to(device=q.device, dtype=torch.int32).contiguous()
        o = torch.empty_like(q)
        lse = torch.empty((batch, heads, n), dtype=torch.float32, device=q.device)
        fwd = nb.nb_attn_fwd_causal if causal else nb.nb_attn_fwd
        fwd(q, k, v, o, lse, lengths, batch, heads, n, d, R, _dtype_code(q),
            torch.cuda.current_stream(q.device))
        ctx.save_for_backward(q, k, v, o, lse, lengths)
        ctx.R = R
        ctx.causal = causal
        return o

    @staticmethod
    def backward(ctx, do):
        q, k, v, o, lse, lengths = ctx.saved_tensors
        batch, heads, n, d = q.shape
        do = do.to(q.dtype).contiguous()
        code = _dtype_code(q)
        ws_bytes = nb.attn_bwd_workspace_size(batch, heads, n, d, code)
        ws = torch.empty(max(ws_bytes, 1), dtype=torch.uint8, device=q.device)
        dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
        bwd = nb.nb_attn_bwd_causal if ctx.causal else nb.nb_attn_bwd
        bwd(q, k, v, o, do, lse, lengths, dq, dk, dv, ws, ws_bytes, batch, heads, n, d, ctx.R, code,
            torch.cuda.current_stream(q.device))
        return dq, dk, dv, None, None, None


def block_sparse_local_attention(q, k, v, lengths=None, R: int = 1, causal: bool = False):
    """Differentiable banded block-sparse local attention (see the class)."""
    return BlockSparseLocalAttention.apply(q, k, v, lengths, R, causal)
