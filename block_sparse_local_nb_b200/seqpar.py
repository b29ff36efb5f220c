"""Sequence parallelism for sequences too long for one GPU: each rank holds a
contiguous shard of the sequence and exchanges halos with its neighbours.

The band is local (NucleoByte page, section 3 "Localized Block-Sparse
Attention Matrix": query block i only sees key blocks |i - j| <= R), so a
shard's outputs depend on at most R blocks (R * 32 rows) on each side of it.
The forward therefore needs a halo of K and V rows from each neighbour; the
backward (section 3 "Custom Backpropagation": P recomputed from the stored
log-sum-exp, D_i = sum_k dO_ik O_ik) needs a halo of Q, K, V, O, dO and lse,
because the keys of the shard are seen by the queries of the halo.  Each rank
then runs the ordinary single-GPU calls on [left halo | shard | right halo]
and keeps the shard's rows: every row of the shard sees exactly the keys (and,
for dK/dV, exactly the queries) it sees in the whole sequence, with the
halo's log-sum-exp and row term taken from the rank that owns those rows.

The exchange is point-to-point (``torch.distributed`` isend/irecv into this
GPU's own memory; NCCL on GPUs, gloo on CPU).  The attention itself runs
through the C ABI by default; ``fwd_fn`` / ``bwd_fn`` replace it (the CPU
tests pass the fp64 reference there).  Layout as everywhere in this library:
[batch, heads, n, d], the sequence on dim 2; ``lengths`` are the sequences'
global lengths.
"""

from __future__ import annotations

import torch
import torch.distributed as dist

BLOCK = 32


def shard_bounds(n: int, world: int, rank: int, align: int = 256) -> tuple[int, int]:
    """[start, end) rows of `rank`'s shard of an n-row sequence: contiguous,
    multiples of `align` rows (a multiple of the 32-row block) except possibly
    the last, as equal as the alignment allows."""
    if n % BLOCK or align % BLOCK or world < 1 or not 0 <= rank < world:
        raise ValueError("n and align must be multiples of 32, 0 <= rank < world")
    units = -(-n // align)
    lo = units * rank // world
    hi = units * (rank + 1) // world
    return min(lo * align, n), min(hi * align, n)


def halo_rows(R: int) -> int:
    """Rows of halo needed on each side: R blocks."""
    return R * BLOCK


def local_lengths(lengths: torch.Tensor, first_row: int, rows: int) -> torch.Tensor:
    """Global sequence lengths seen from a buffer whose row 0 is global row
    `first_row` and that holds `rows` rows (clamped to [0, rows])."""
    return (lengths.to(torch.int64) - first_row).clamp(0, rows).to(torch.int32)


def halo_slices(full: torch.Tensor, start: int, end: int, h: int):
    """The halos of the shard [start, end) cut from a whole-sequence tensor
    (what exchange_halo delivers, for callers that hold every shard)."""
    n = full.shape[2]
    return full[:, :, max(0, start - h):start], full[:, :, end:min(n, end + h)]


def exchange_halo(t: torch.Tensor, h: int, rank: int, world: int, group=None):
    """The `h` rows before and after this rank's shard `t` (sequence on dim 2),
    received from the neighbouring ranks (empty at the sequence's ends).  Every
    rank sends its first `h` rows to the left neighbour and its last `h` rows
    to the right neighbour.  Every shard but the last must hold at least `h`
    rows."""
    empty = t[:, :, :0]
    if world == 1 or h == 0:
        return empty, empty
    if t.shape[2] < h:
        raise ValueError("a shard must hold at least the halo's rows")
    left = torch.empty_like(t[:, :, :h]) if rank > 0 else empty
    right = torch.empty_like(t[:, :, :h]) if rank < world - 1 else empty
    ops = []
    if rank > 0:
        ops.append(dist.P2POp(dist.isend, t[:, :, :h].contiguous(), rank - 1, group))
        ops.append(dist.P2POp(dist.irecv, left, rank - 1, group))
    if rank < world - 1:
        ops.append(dist.P2POp(dist.isend, t[:, :, -h:].contiguous(), rank + 1, group))
        ops.append(dist.P2POp(dist.irecv, right, rank + 1, group))
    for req in dist.batch_isend_irecv(ops):
        req.wait()
    return left, right


def _extend(t, left, right):
    return torch.cat([left, t, right], dim=2).contiguous()


def _native_fwd(q, k, v, lengths, R, causal):
    from . import binding as nb

    batch, heads, n, d = q.shape
    o = torch.empty_like(q)
    lse = torch.empty((batch, heads, n), dtype=torch.float32, device=q.device)
    dtype = nb.NB_BF16 if q.dtype == torch.bfloat16 else nb.NB_F32
    fwd = nb.nb_attn_fwd_causal if causal else nb.nb_attn_fwd
    fwd(q, k, v, o, lse, lengths, batch, heads, n, d, R, dtype)
    return o, lse


def _native_bwd(q, k, v, o, do, lse, lengths, R, causal):
    from . import binding as nb

    batch, heads, n, d = q.shape
    dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
    ws_bytes = nb.attn_bwd_workspace_size(batch, heads, n, d, nb.NB_BF16)
    ws = torch.empty(max(ws_bytes, 1), dtype=torch.uint8, device=q.device)
    bwd = nb.nb_attn_bwd_causal if causal else nb.nb_attn_bwd
    bwd(q, k, v, o, do, lse, lengths, dq, dk, dv, ws, ws_bytes, batch, heads, n, d, R, nb.NB_BF16)
    return dq, dk, dv


def fwd_with_halo(q, k, v, k_halo, v_halo, lengths, R: int, start: int, causal: bool = False,
                  fwd_fn=None):
    """Forward of the shard whose first row is global row `start`, given the
    (left, right) halos of K and V.  Returns (O, lse) of the shard's rows."""
    (kl, kr), (vl, vr) = k_halo, v_halo
    ql, qr = q.new_zeros(kl.shape), q.new_zeros(kr.shape)  # halo queries: outputs dropped
    ext = [_extend(q, ql, qr), _extend(k, kl, kr), _extend(v, vl, vr)]
    lens = local_lengths(lengths, start - kl.shape[2], ext[0].shape[2]).to(q.device)
    o, lse = (fwd_fn or _native_fwd)(*ext, lens, R, causal)
    a, b = kl.shape[2], kl.shape[2] + q.shape[2]
    return o[:, :, a:b].contiguous(), lse[:, :, a:b].contiguous()


def bwd_with_halo(q, k, v, o, do, lse, halos, lengths, R: int, start: int, causal: bool = False,
                  bwd_fn=None):
    """Backward of the shard whose first row is global row `start`, given the
    (left, right) halos of Q, K, V, O, dO and lse in ``halos`` (a dict keyed by
    those names).  Returns (dQ, dK, dV) of the shard's rows."""
    ext = {name: _extend(t, *halos[name]) for name, t in
           (("q", q), ("k", k), ("v", v), ("o", o), ("do", do))}
    lse_ext = torch.cat([halos["lse"][0], lse, halos["lse"][1]], dim=2).contiguous()
    left = halos["q"][0].shape[2]
    lens = local_lengths(lengths, start - left, ext["q"].shape[2]).to(q.device)
    grads = (bwd_fn or _native_bwd)(ext["q"], ext["k"], ext["v"], ext["o"], ext["do"], lse_ext,
                                     lens, R, causal)
    return tuple(t[:, :, left:left + q.shape[2]].contiguous() for t in grads)


def seqpar_attn_fwd(q, k, v, lengths, R: int, start: int, rank: int, world: int, group=None,
                    causal: bool = False, fwd_fn=None):
    """Forward of this rank's shard (rows [start, start + q.shape[2]) of the
    sequence): exchange the K/V halos, then fwd_with_halo."""
    h = halo_rows(R)
    k_halo = exchange_halo(k, h, rank, world, group)
    v_halo = exchange_halo(v, h, rank, world, group)
    return fwd_with_halo(q, k, v, k_halo, v_halo, lengths, R, start, causal, fwd_fn)


def seqpar_attn_bwd(q, k, v, o, do, lse, lengths, R: int, start: int, rank: int, world: int,
                    group=None, causal: bool = False, bwd_fn=None):
    """Backward of this rank's shard: exchange the Q, K, V, O, dO and lse
    halos, then bwd_with_halo."""
    h = halo_rows(R)
    halos = {name: exchange_halo(t, h, rank, world, group)
             for name, t in (("q", q), ("k", k), ("v", v), ("o", o), ("do", do))}
    l_, r_ = exchange_halo(lse.unsqueeze(-1), h, rank, world, group)
    halos["lse"] = (l_.squeeze(-1), r_.squeeze(-1))
    return bwd_with_halo(q, k, v, o, do, lse, halos, lengths, R, start, causal, bwd_fn)
