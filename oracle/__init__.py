"""Plain, slow, obviously correct CPU oracle for the banded block-sparse local
attention (forward and backward) and the 2-bit DNA k-mer tokenizer.

TEST INFRASTRUCTURE ONLY.  Nothing in the product path imports, links or calls
this package: only ``tests/``, ``__graft_entry__.smoke()`` and ``bench.py``'s
CPU-baseline leg (and its ``--impl reference`` arm) may use it.  It shares no
code, table or constant generator with the CUDA library.

Source of the method: the NucleoByte page ("NucleoByte: GPU-Accelerated
Block-Sparse Genomic Language Model"), section 3 "Mathematical Foundations"
(band predicate, scaled scores, online-softmax updates, backward row term D_i
and softmax gradient) and sections 1, 2 and 5 (2-bit k-mer tokenizer, padding
to a multiple of 32, the worked k-mer example).

All floating point is fp64 (NumPy).  Every function is pinned by a CPU test in
``tests/test_oracle_*.py`` against something other than itself (brute force,
closed forms, invariants, finite differences, values printed on the page).
"""

from .attention import (  # noqa: F401
    BLOCK,
    block_band_mask,
    attn_fwd_dense,
    attn_bwd_dense,
    attn_fwd_banded,
    attn_bwd_banded,
    attn_bwd_from_saved,
)
from .tokenizer import kmer_ids, pack_2bit, N_FLAG_BASE  # noqa: F401
