"""Host-side logic of the training-layer glue (no GPU): the dynamic-ceiling
layout of a batch, checked against the oracle's ceiling and window counts."""

import numpy as np
import pytest

from block_sparse_local_nb_b200.layer import ceiling_layout
from oracle.tokenizer import ceiling, kmer_ids


@pytest.mark.parametrize("counts,k", [([30], 6), ([0, 5, 6, 37], 6), ([4101] * 3, 6),
                                      ([1, 2, 3], 1), ([], 6), ([100, 4200, 7], 7)])
def test_ceiling_layout_matches_oracle(counts, k):
    offsets, n_pad = ceiling_layout(counts, k)
    assert offsets.tolist() == [0] + np.cumsum(counts, dtype=np.int64).tolist()
    windows = [kmer_ids(b"A" * c, k).shape[0] for c in counts]
    assert n_pad == ceiling(max(windows, default=0))
    assert n_pad % 32 == 0 and all(w <= n_pad for w in windows)


def test_ceiling_layout_rejects_negative_counts():
    with pytest.raises(ValueError):
        ceiling_layout([3, -1])
