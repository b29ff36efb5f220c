"""Host-side logic of the training-layer glue (no GPU): the dynamic-ceiling
layout of a batch, computed by the library's host-only nb_batch_ceiling and
checked against the oracle's ceiling and window counts."""

import ctypes

import numpy as np
import pytest

from block_sparse_local_nb_b200 import binding
from block_sparse_local_nb_b200.layer import ceiling_layout
from oracle.tokenizer import ceiling, kmer_ids

NB_ERR_INVALID_ARG, NB_ERR_UNSUPPORTED = -1, -2


@pytest.mark.parametrize("counts,k", [([30], 6), ([0, 5, 6, 37], 6), ([4101] * 3, 6),
                                      ([1, 2, 3], 1), ([], 6), ([100, 4200, 7], 7),
                                      ([37, 38, 32], 6), ([5], 6)])
def test_ceiling_layout_matches_oracle(built_lib, counts, k):
    offsets, n_pad = ceiling_layout(counts, k)
    assert offsets.tolist() == [0] + np.cumsum(counts, dtype=np.int64).tolist()
    windows = [kmer_ids(b"A" * c, k).shape[0] for c in counts]
    assert n_pad == ceiling(max(windows, default=0))
    assert n_pad % 32 == 0 and all(w <= n_pad for w in windows)


def test_ceiling_layout_rejects_negative_counts(built_lib):
    with pytest.raises(ValueError):
        ceiling_layout([3, -1])


def test_batch_ceiling_decreasing_offsets_are_empty(built_lib):
    # sequence 1 has offsets going backwards: no bases, no windows
    assert binding.nb_batch_ceiling([0, 100, 50, 90], 3, 6) == ceiling(95)
    assert binding.nb_batch_ceiling([10, 5], 1, 6) == 0


def test_batch_ceiling_rejects_bad_arguments(built_lib):
    out = ctypes.c_int32(-7)
    off = (ctypes.c_int64 * 2)(0, 100)
    assert built_lib.nb_batch_ceiling(off, 1, 0, ctypes.byref(out)) == NB_ERR_UNSUPPORTED
    assert built_lib.nb_batch_ceiling(off, 1, 8, ctypes.byref(out)) == NB_ERR_UNSUPPORTED
    assert built_lib.nb_batch_ceiling(off, -1, 6, ctypes.byref(out)) == NB_ERR_INVALID_ARG
    assert built_lib.nb_batch_ceiling(None, 1, 6, ctypes.byref(out)) == NB_ERR_INVALID_ARG
    assert built_lib.nb_batch_ceiling(off, 1, 6, None) == NB_ERR_INVALID_ARG
    big = (ctypes.c_int64 * 2)(0, 1 << 40)  # more windows than an int32 width holds
    assert built_lib.nb_batch_ceiling(big, 1, 6, ctypes.byref(out)) == NB_ERR_INVALID_ARG
    assert out.value == -7  # not written on error
    assert built_lib.nb_batch_ceiling(None, 0, 6, ctypes.byref(out)) == 0 and out.value == 0
