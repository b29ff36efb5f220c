"""Thin ctypes binding of the C ABI in ``include/nb.h`` (argument marshalling only).

Functions carry the C names and accept torch tensors (their ``data_ptr()`` is
passed) or raw integer addresses.  Every step of the computation runs in
``libnb_b200.so``; there is no fallback: if the library is missing the first
call raises.  A non-zero status raises :class:`NbError`.
"""

from __future__ import annotations

import ctypes
import os
import threading

NB_F32 = 0
NB_BF16 = 1

_LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libnb_b200.so")
_lock = threading.Lock()
_lib = None

# (name, restype, argtypes) for every function declared in include/nb.h
_P = ctypes.c_void_p
_I = ctypes.c_int
_SIGS = [
    ("nb_status_string", ctypes.c_char_p, [_I]),
    ("nb_abi_version", _I, []),
    ("nb_kernel_error", _I, [ctypes.POINTER(ctypes.c_int), _I]),
    ("nb_attn_fwd", _I, [_P, _P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _I, _P]),
    ("nb_attn_fwd_causal", _I, [_P, _P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _I, _P]),
    ("nb_attn_bwd_workspace_size", ctypes.c_size_t, [_I, _I, _I, _I, _I]),
    ("nb_attn_bwd", _I, [_P, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P, ctypes.c_size_t,
                         _I, _I, _I, _I, _I, _I, _P]),
    ("nb_attn_bwd_causal", _I, [_P, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P, ctypes.c_size_t,
                                _I, _I, _I, _I, _I, _I, _P]),
    ("nb_attn_fwd_bwd_host_workspace_size", ctypes.c_size_t, [_I, _I, _I, _I, _I, _I]),
    ("nb_attn_fwd_bwd_host", _I, [_P] * 11 + [ctypes.c_size_t] + [_I] * 7 + [_P]),
    ("nb_tokenize_kmer", _I, [_P, ctypes.c_int64, _P, _P, _I, _P]),
    ("nb_tokenize_batch", _I, [_P, _P, _I, _I, _P, _P, _I, _P]),
    ("nb_batch_ceiling", _I, [_P, _I, _I, ctypes.POINTER(ctypes.c_int32)]),
]


class NbError(RuntimeError):
    def __init__(self, status: int, what: str):
        self.status = status
        super().__init__(f"{what} failed: {nb_status_string(status)} ({status})")


def lib() -> ctypes.CDLL:
    """Load libnb_b200.so once; raise if it has not been built."""
    global _lib
    if _lib is None:
        with _lock:
            if _lib is None:
                if not os.path.exists(_LIB_PATH):
                    raise RuntimeError(
                        f"{_LIB_PATH} is missing: build it with "
                        "`python -m block_sparse_local_nb_b200.build` (no CPU fallback exists)")
                cdll = ctypes.CDLL(_LIB_PATH)
                for name, res, args in _SIGS:
                    fn = getattr(cdll, name)
                    fn.restype = res
                    fn.argtypes = args
                _lib = cdll
    return _lib


def _ptr(x):
    if x is None:
        return None
    if isinstance(x, int):
        return x
    return x.data_ptr()


def _stream(stream):
    if stream is None:
        import torch

        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, int):
        return stream
    return stream.cuda_stream


def _check(status: int, what: str):
    if status != 0:
        raise NbError(status, what)


def nb_kernel_error(clear: bool = True) -> int:
    """Synchronise the device and return the first recorded kernel wait-timeout code (0 = none)."""
    code = ctypes.c_int(0)
    _check(lib().nb_kernel_error(ctypes.byref(code), 1 if clear else 0), "nb_kernel_error")
    return code.value


def nb_status_string(status: int) -> str:
    return lib().nb_status_string(status).decode()


def nb_attn_fwd(q, k, v, o, lse, lengths, batch, heads, n, d, R, dtype, stream=None, check=True):
    st = lib().nb_attn_fwd(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), _ptr(lengths),
                           batch, heads, n, d, R, dtype, _stream(stream))
    if check:
        _check(st, "nb_attn_fwd")
    return st


def nb_attn_fwd_causal(q, k, v, o, lse, lengths, batch, heads, n, d, R, dtype, stream=None,
                       check=True):
    st = lib().nb_attn_fwd_causal(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), _ptr(lengths),
                                  batch, heads, n, d, R, dtype, _stream(stream))
    if check:
        _check(st, "nb_attn_fwd_causal")
    return st


def attn_bwd_workspace_size(batch, heads, n, d, dtype) -> int:
    return int(lib().nb_attn_bwd_workspace_size(batch, heads, n, d, dtype))


def nb_attn_bwd(q, k, v, o, dout, lse, lengths, dq, dk, dv, workspace, workspace_bytes,
                batch, heads, n, d, R, dtype, stream=None, check=True):
    st = lib().nb_attn_bwd(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(dout), _ptr(lse),
                           _ptr(lengths), _ptr(dq), _ptr(dk), _ptr(dv), _ptr(workspace),
                           workspace_bytes, batch, heads, n, d, R, dtype, _stream(stream))
    if check:
        _check(st, "nb_attn_bwd")
    return st


def nb_attn_bwd_causal(q, k, v, o, dout, lse, lengths, dq, dk, dv, workspace, workspace_bytes,
                       batch, heads, n, d, R, dtype, stream=None, check=True):
    st = lib().nb_attn_bwd_causal(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(dout), _ptr(lse),
                                  _ptr(lengths), _ptr(dq), _ptr(dk), _ptr(dv), _ptr(workspace),
                                  workspace_bytes, batch, heads, n, d, R, dtype, _stream(stream))
    if check:
        _check(st, "nb_attn_bwd_causal")
    return st


def attn_fwd_bwd_host_workspace_size(batch, heads, n, d, R, dtype) -> int:
    return int(lib().nb_attn_fwd_bwd_host_workspace_size(batch, heads, n, d, R, dtype))


def nb_attn_fwd_bwd_host(q, k, v, dout, lengths, o, lse, dq, dk, dv, workspace, workspace_bytes,
                         batch, heads, n, d, R, dtype, causal=False, stream=None, check=True):
    """Forward + backward of HOST tensors (pinned CPU tensors or addresses); the
    workspace is a device buffer.  Asynchronous on `stream`."""
    st = lib().nb_attn_fwd_bwd_host(_ptr(q), _ptr(k), _ptr(v), _ptr(dout), _ptr(lengths),
                                    _ptr(o), _ptr(lse), _ptr(dq), _ptr(dk), _ptr(dv),
                                    _ptr(workspace), workspace_bytes, batch, heads, n, d, R,
                                    dtype, 1 if causal else 0, _stream(stream))
    if check:
        _check(st, "nb_attn_fwd_bwd_host")
    return st


def nb_tokenize_kmer(seq, length, ids, packed, k=6, stream=None, check=True):
    st = lib().nb_tokenize_kmer(_ptr(seq), length, _ptr(ids), _ptr(packed), k, _stream(stream))
    if check:
        _check(st, "nb_tokenize_kmer")
    return st


def nb_tokenize_batch(seqs, offsets, batch, k, input_ids, lengths, n_pad, stream=None, check=True):
    st = lib().nb_tokenize_batch(_ptr(seqs), _ptr(offsets), batch, k, _ptr(input_ids),
                                 _ptr(lengths), n_pad, _stream(stream))
    if check:
        _check(st, "nb_tokenize_batch")
    return st


def nb_batch_ceiling(offsets, batch, k=6) -> int:
    """The dynamic ceiling (n_pad) of a batch from its HOST int64 offsets
    [batch + 1] (a NumPy array or a sequence of ints)."""
    import numpy as np

    off = np.ascontiguousarray(np.asarray(offsets, dtype=np.int64))
    if off.size < batch + 1:
        raise ValueError("offsets must hold batch + 1 entries")
    out = ctypes.c_int32(0)
    st = lib().nb_batch_ceiling(off.ctypes.data if off.size else None, batch, k, ctypes.byref(out))
    _check(st, "nb_batch_ceiling")
    return int(out.value)
