"""Helpers for the GPU parity tests: run the CUDA library through its C ABI on
torch-owned device memory and compare with the CPU oracle."""

import numpy as np
import torch

import block_sparse_local_nb_b200 as nb

BLOCK = 32
O_ATOL_BF16 = 1.5e-2   # max-abs on O (bf16)
LSE_ATOL_BF16 = 1e-3   # max-abs on log-sum-exp (bf16 inputs, fp32 arithmetic)
GRAD_RFRO_BF16 = 1e-2  # relative Frobenius on dQ, dK, dV (bf16)
ATOL_F32 = 1e-4        # max-abs on O and log-sum-exp (fp32)


def dtype_code(t: torch.dtype) -> int:
    return nb.NB_F32 if t == torch.float32 else nb.NB_BF16


def run_fwd(q, k, v, lengths, R, with_lse=True, causal=False):
    """Forward through nb_attn_fwd (or nb_attn_fwd_causal); returns (o, lse) device tensors."""
    batch, heads, n, d = q.shape
    o = torch.empty_like(q)
    lse = torch.empty((batch, heads, n), device=q.device, dtype=torch.float32) if with_lse else None
    lens = None if lengths is None else lengths.to(device=q.device, dtype=torch.int32)
    fwd = nb.nb_attn_fwd_causal if causal else nb.nb_attn_fwd
    fwd(q, k, v, o, lse, lens, batch, heads, n, d, R, dtype_code(q.dtype))
    return o, lse


def run_bwd(q, k, v, o, do, lse, lengths, R, workspace=None, causal=False):
    batch, heads, n, d = q.shape
    dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
    ws_bytes = nb.attn_bwd_workspace_size(batch, heads, n, d, dtype_code(q.dtype))
    if workspace is None:
        workspace = torch.empty(max(ws_bytes, 1), dtype=torch.uint8, device=q.device)
    lens = None if lengths is None else lengths.to(device=q.device, dtype=torch.int32)
    bwd = nb.nb_attn_bwd_causal if causal else nb.nb_attn_bwd
    bwd(q, k, v, o, do, lse, lens, dq, dk, dv, workspace, ws_bytes, batch, heads, n, d, R,
        dtype_code(q.dtype))
    return dq, dk, dv


def f64(t) -> np.ndarray:
    return t.detach().to("cpu", torch.float64).numpy()


def max_abs(a, b) -> float:
    a, b = np.asarray(a, np.float64), np.asarray(b, np.float64)
    both_inf = np.isinf(a) & np.isinf(b) & (np.sign(a) == np.sign(b))
    with np.errstate(invalid="ignore"):
        diff = np.where(both_inf, 0.0, np.abs(a - b))
    return float(diff.max()) if diff.size else 0.0


def rel_fro(got, want) -> float:
    got, want = np.asarray(got, np.float64), np.asarray(want, np.float64)
    den = np.linalg.norm(want)
    num = np.linalg.norm(got - want)
    return float(num / den) if den > 0 else float(num)


def window(n_blocks, lo, hi, R):
    """Block range [s, e) of a sub-sequence on which the oracle's outputs for
    query/key blocks [lo, hi) are exact: two band radii of context each side."""
    return max(0, lo - 2 * R), min(n_blocks, hi + 2 * R)
