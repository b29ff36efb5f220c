"""CPU checks of the C-ABI library: it loads, exports every function that
include/nb.h declares, and rejects invalid arguments on the host (these calls
return before any CUDA call, so they run without a GPU)."""

import ctypes
import os
import re
import subprocess

import pytest

from tests.conftest import ROOT

HEADER = os.path.join(ROOT, "include", "nb.h")
LIB = os.path.join(ROOT, "block_sparse_local_nb_b200", "libnb_b200.so")

NB_OK, NB_ERR_INVALID_ARG, NB_ERR_UNSUPPORTED, NB_ERR_MISALIGNED = 0, -1, -2, -3
NB_ERR_WORKSPACE = -5
F32, BF16 = 0, 1


def _declared_functions():
    text = open(HEADER).read()
    return sorted(set(re.findall(r"NB_API\s+[\w\s\*]+?\b(nb_\w+)\s*\(", text)))


@pytest.fixture(scope="module")
def lib():
    if not os.path.exists(LIB):
        from block_sparse_local_nb_b200.build import build

        build()
    from block_sparse_local_nb_b200 import binding

    return binding.lib()


def test_header_declares_the_abi():
    names = _declared_functions()
    assert {"nb_attn_fwd", "nb_attn_bwd", "nb_attn_bwd_workspace_size", "nb_tokenize_kmer",
            "nb_status_string", "nb_abi_version"} <= set(names)


def test_library_exports_every_declared_symbol(lib):
    out = subprocess.run(["nm", "-D", "--defined-only", LIB], capture_output=True, text=True,
                         check=True).stdout
    exported = set(re.findall(r"\sT\s(nb_\w+)", out))
    for name in _declared_functions():
        assert name in exported, name
        assert getattr(lib, name) is not None


def test_library_links_no_cuda_runtime_dynamically():
    out = subprocess.run(["ldd", LIB], capture_output=True, text=True).stdout
    assert "libcudart" not in out and "libtorch" not in out


def test_status_strings(lib):
    for st in (0, -1, -2, -3, -4, -5, -6):
        assert lib.nb_status_string(st)
    assert lib.nb_abi_version() >= 100


def _fwd(lib, q=16, k=16, v=16, o=16, lse=None, lengths=None, batch=1, heads=1, n=64, d=64,
         R=1, dtype=BF16):
    return lib.nb_attn_fwd(q, k, v, o, lse, lengths, batch, heads, n, d, R, dtype, None)


@pytest.mark.parametrize("kw,status", [
    (dict(n=48), NB_ERR_INVALID_ARG),        # n not a multiple of 32
    (dict(n=-32), NB_ERR_INVALID_ARG),
    (dict(R=-1), NB_ERR_INVALID_ARG),
    (dict(batch=-1), NB_ERR_INVALID_ARG),
    (dict(dtype=7), NB_ERR_INVALID_ARG),
    (dict(d=32), NB_ERR_UNSUPPORTED),
    (dict(d=96), NB_ERR_UNSUPPORTED),
    (dict(q=None), NB_ERR_INVALID_ARG),
    (dict(o=None), NB_ERR_INVALID_ARG),
    (dict(k=24), NB_ERR_MISALIGNED),
    (dict(lse=20), NB_ERR_MISALIGNED),
    (dict(lengths=18), NB_ERR_MISALIGNED),
    (dict(heads=70000), NB_ERR_UNSUPPORTED),
])
def test_fwd_rejects_invalid_arguments(lib, kw, status):
    assert _fwd(lib, **kw) == status


def test_fwd_empty_problem_is_a_no_op(lib):
    assert _fwd(lib, batch=0) == NB_OK
    assert _fwd(lib, heads=0, q=None, k=None, v=None, o=None) == NB_OK
    assert _fwd(lib, n=0) == NB_OK


def test_bwd_workspace_size(lib):
    ws = lib.nb_attn_bwd_workspace_size(4, 12, 4096, 64, BF16)
    rows = 4 * 12 * 4096
    # row term D, -lse*log2(e) and the fp32 dQ accumulator, each 256-byte aligned
    assert ws >= 2 * rows * 4 + rows * 64 * 4
    assert ws < 2 * rows * 4 + rows * 64 * 4 + 3 * 256
    assert lib.nb_attn_bwd_workspace_size(1, 1, 33, 64, BF16) == 0  # invalid n
    assert lib.nb_attn_bwd_workspace_size(0, 1, 64, 64, BF16) == 0


def _bwd(lib, ws=256, ws_bytes=1 << 30, dq=16, lse=16, dtype=BF16, n=64, d=64, R=1, k=16):
    return lib.nb_attn_bwd(16, k, 16, 16, 16, lse, None, dq, 16, 16, ws, ws_bytes, 1, 1, n, d, R,
                           dtype, None)


@pytest.mark.parametrize("kw,status", [
    (dict(ws=None), NB_ERR_WORKSPACE),
    (dict(ws=272), NB_ERR_WORKSPACE),       # not 256-byte aligned
    (dict(ws_bytes=100), NB_ERR_WORKSPACE),  # too small
    (dict(lse=None), NB_ERR_INVALID_ARG),
    (dict(dq=None), NB_ERR_INVALID_ARG),
    (dict(dq=8), NB_ERR_MISALIGNED),
    (dict(k=40), NB_ERR_MISALIGNED),
    (dict(dtype=F32), NB_ERR_UNSUPPORTED),
    (dict(n=40), NB_ERR_INVALID_ARG),
    (dict(R=-2), NB_ERR_INVALID_ARG),
])
def test_bwd_rejects_invalid_arguments(lib, kw, status):
    assert _bwd(lib, **kw) == status


@pytest.mark.parametrize("args,status", [
    ((16, -1, 32, None, 6), NB_ERR_INVALID_ARG),
    ((16, 100, 32, None, 0), NB_ERR_UNSUPPORTED),
    ((16, 100, 32, None, 8), NB_ERR_UNSUPPORTED),
    ((16, 100, 33, None, 6), NB_ERR_MISALIGNED),
    ((None, 100, 32, None, 6), NB_ERR_INVALID_ARG),
    ((16, 0, 32, 32, 6), NB_OK),
    ((16, 100, None, None, 6), NB_OK),
    ((16, 5, 32, None, 6), NB_OK),  # len < k with only ids: nothing to write
])
def test_tokenize_rejects_invalid_arguments(lib, args, status):
    seq, n, ids, packed, k = args
    assert lib.nb_tokenize_kmer(seq, n, ids, packed, k, None) == status


@pytest.mark.parametrize("kw,status", [
    (dict(batch=-1), NB_ERR_INVALID_ARG),
    (dict(n_pad=48), NB_ERR_INVALID_ARG),       # not a multiple of 32
    (dict(n_pad=-32), NB_ERR_INVALID_ARG),
    (dict(k=0), NB_ERR_UNSUPPORTED),
    (dict(k=8), NB_ERR_UNSUPPORTED),
    (dict(batch=70000), NB_ERR_UNSUPPORTED),
    (dict(seqs=None), NB_ERR_INVALID_ARG),
    (dict(offsets=None), NB_ERR_INVALID_ARG),
    (dict(ids=None), NB_ERR_INVALID_ARG),
    (dict(ids=40), NB_ERR_MISALIGNED),
    (dict(offsets=12), NB_ERR_MISALIGNED),
    (dict(lengths=18), NB_ERR_MISALIGNED),
    (dict(batch=0), NB_OK),
    (dict(n_pad=0, lengths=None), NB_OK),
])
def test_tokenize_batch_rejects_invalid_arguments(lib, kw, status):
    args = dict(seqs=16, offsets=16, batch=2, k=6, ids=16, lengths=16, n_pad=64)
    args.update(kw)
    assert lib.nb_tokenize_batch(args["seqs"], args["offsets"], args["batch"], args["k"], args["ids"],
                                 args["lengths"], args["n_pad"], None) == status


@pytest.mark.parametrize("kw,status", [
    (dict(n=48), NB_ERR_INVALID_ARG), (dict(R=-1), NB_ERR_INVALID_ARG), (dict(d=96), NB_ERR_UNSUPPORTED),
    (dict(k=24), NB_ERR_MISALIGNED), (dict(batch=0), NB_OK),
])
def test_causal_entry_points_validate_like_the_band(lib, kw, status):
    args = dict(q=16, k=16, v=16, o=16, lse=None, lengths=None, batch=1, heads=1, n=64, d=64, R=1,
                dtype=BF16)
    args.update(kw)
    a = args
    assert lib.nb_attn_fwd_causal(a["q"], a["k"], a["v"], a["o"], a["lse"], a["lengths"], a["batch"],
                                  a["heads"], a["n"], a["d"], a["R"], a["dtype"], None) == status
    st = lib.nb_attn_bwd_causal(a["q"], a["k"], a["v"], a["o"], 16, 16, None, 16, 16, 16, 256,
                                1 << 30, a["batch"], a["heads"], a["n"], a["d"], a["R"], a["dtype"],
                                None)
    assert st == status


def test_causal_backward_rejects_fp32(lib):
    assert lib.nb_attn_bwd_causal(16, 16, 16, 16, 16, 16, None, 16, 16, 16, 256, 1 << 30, 1, 1, 64,
                                  64, 1, F32, None) == NB_ERR_UNSUPPORTED


def test_noalloc_rejects_on_the_host(lib):
    """nb_attn_bwd_noalloc checks shape, dtype, its scratch limit and pointers
    before it touches the device: these calls return without a GPU."""
    fn = lib.nb_attn_bwd_noalloc
    fn.restype = ctypes.c_int
    fn.argtypes = [ctypes.c_void_p] * 10 + [ctypes.c_int] * 6 + [ctypes.c_void_p]
    nulls = [None] * 10
    # 1 x 8 x 65536 x 64 needs about 130 MiB of scratch, beyond the 64 MiB array
    assert fn(*nulls, 1, 8, 65536, 64, 1, BF16, None) == NB_ERR_WORKSPACE
    assert fn(*nulls, 1, 1, 64, 64, 1, F32, None) == NB_ERR_UNSUPPORTED
    assert fn(*nulls, 1, 1, 48, 64, 1, BF16, None) == NB_ERR_INVALID_ARG
    assert fn(*nulls, 1, 1, 64, 64, 1, BF16, None) == NB_ERR_INVALID_ARG  # null pointers
    assert fn(*nulls, 0, 1, 64, 64, 1, BF16, None) == NB_OK  # empty problem
    ptrs = [16] * 6 + [None] + [16, 16, 24]  # dv not 16-byte aligned
    assert fn(*ptrs, 1, 1, 64, 64, 1, BF16, None) == NB_ERR_MISALIGNED


_HOST_BUF = ctypes.create_string_buffer(4096)  # real host memory for the host-side tensors
_HB = ctypes.addressof(_HOST_BUF)


def _host(lib, ws=None, ws_bytes=1 << 40, q=_HB, dq=_HB, dtype=BF16, n=64, d=64, R=1, batch=1):
    """Every case is rejected before any copy or launch; the workspace (the only
    device pointer) is NULL unless the case is about the workspace, so a change
    in the order of the checks fails here on the host."""
    fn = lib.nb_attn_fwd_bwd_host
    return fn(q, _HB, _HB, _HB, None, _HB, None, dq, _HB, _HB, ws, ws_bytes, batch, 2, n, d, R,
              dtype, 0, None)


@pytest.mark.parametrize("kw,status", [
    (dict(q=None), NB_ERR_INVALID_ARG),
    (dict(dq=None), NB_ERR_INVALID_ARG),
    (dict(n=40), NB_ERR_INVALID_ARG),
    (dict(R=-1), NB_ERR_INVALID_ARG),
    (dict(d=96), NB_ERR_UNSUPPORTED),
    (dict(dtype=F32), NB_ERR_UNSUPPORTED),
    (dict(ws=None), NB_ERR_WORKSPACE),
    (dict(ws=272), NB_ERR_WORKSPACE),
    (dict(ws_bytes=1024), NB_ERR_WORKSPACE),
    (dict(batch=0), NB_OK),
])
def test_host_step_rejects_invalid_arguments(lib, kw, status):
    assert _host(lib, **kw) == status


def test_host_step_workspace_holds_a_few_chunks(lib):
    """The host entry point's device scratch holds three chunks, not the whole
    problem: 1 x 8 x 2^20 x 64 at R = 8 has eight slices, each cut into four
    windows that own 8192 blocks and carry 2R = 16 blocks of context a side."""
    n, d, R = 1 << 20, 64, 8
    ws = lib.nb_attn_fwd_bwd_host_workspace_size(1, 8, n, d, R, BF16)
    rows = (8192 + 4 * R) * 32  # an inner window
    one = 8 * rows * d * 2 + rows * 4 + lib.nb_attn_bwd_workspace_size(1, 1, rows, d, BF16)
    assert 3 * one <= ws <= 3 * one + 64 * 1024
    assert lib.nb_attn_fwd_bwd_host_workspace_size(1, 8, n, d, R, F32) == 0
    assert lib.nb_attn_fwd_bwd_host_workspace_size(0, 8, n, d, R, BF16) == 0
    assert lib.nb_attn_fwd_bwd_host_workspace_size(1, 8, n, d, -1, BF16) == 0
    # a slice too short to cut: one chunk, one slot
    one = lib.nb_attn_fwd_bwd_host_workspace_size(1, 1, 64, d, 1, BF16)
    assert one < 2 * (8 * 64 * d * 2 + 64 * 4 + lib.nb_attn_bwd_workspace_size(1, 1, 64, d, BF16))
