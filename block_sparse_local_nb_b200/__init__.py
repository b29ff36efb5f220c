"""B200-native banded block-sparse local attention and 2-bit k-mer tokenizer.

The compute lives in the CUDA library ``libnb_b200.so`` (C ABI declared in
``include/nb.h``); :mod:`block_sparse_local_nb_b200.binding` marshals arguments
to it.  Importing the package does not load the library; the first call does,
and raises if the library was not built.
"""

from .binding import (  # noqa: F401
    NB_BF16,
    NB_F32,
    NbError,
    attn_bwd_workspace_size,
    attn_fwd_bwd_host_workspace_size,
    lib,
    nb_attn_bwd,
    nb_attn_bwd_causal,
    nb_attn_fwd,
    nb_attn_fwd_bwd_host,
    nb_attn_fwd_causal,
    nb_batch_ceiling,
    nb_kernel_error,
    nb_status_string,
    nb_tokenize_batch,
    nb_tokenize_kmer,
)
