"""GPU checks of the training-layer glue: the collator against the model-ID
oracle (bit-exact) and the autograd function against the direct C-ABI calls
and against the fp64 oracle."""

import numpy as np
import pytest
import torch

import block_sparse_local_nb_b200 as nb
from block_sparse_local_nb_b200.inputs import random_attn_inputs
from block_sparse_local_nb_b200.layer import block_sparse_local_attention, collate
from oracle import attn_bwd_banded, attn_fwd_banded
from oracle.tokenizer import model_ids_batch
from tests.gpu_util import GRAD_RFRO_BF16, O_ATOL_BF16, f64, max_abs, rel_fro, run_bwd, run_fwd

pytestmark = pytest.mark.gpu


def test_collate_matches_oracle():
    rng = np.random.default_rng(8)
    alphabet = np.frombuffer(b"ACGTACGTACGTN", np.uint8)
    seqs = [alphabet[rng.integers(0, alphabet.size, int(n))].tobytes()
            for n in [0, 3, 6, 7, 37, 38, 39] + rng.integers(0, 2000, 25).tolist()]
    ids, lengths = collate(seqs, 6)
    torch.cuda.synchronize()
    want, want_len = model_ids_batch(seqs, 6)
    assert ids.dtype == torch.int64 and ids.shape == want.shape and ids.shape[1] % 32 == 0
    assert np.array_equal(ids.cpu().numpy(), want)
    assert np.array_equal(lengths.cpu().numpy(), want_len)


def test_collate_all_short():
    ids, lengths = collate([b"ACG", b""], 6)
    torch.cuda.synchronize()
    assert ids.shape == (2, 0) and lengths.cpu().tolist() == [0, 0]


def test_autograd_matches_direct_calls():
    q, k, v, do = (t.cuda() for t in random_attn_inputs(2, 3, 512, 64, "bf16", seed=31))
    L = torch.tensor([512, 300], dtype=torch.int32)
    qa, ka, va = (t.clone().requires_grad_(True) for t in (q, k, v))
    o = block_sparse_local_attention(qa, ka, va, L.cuda(), 2)
    o.backward(do)
    o_ref, lse = run_fwd(q, k, v, L, 2)
    dq, dk, dv = run_bwd(q, k, v, o_ref, do, lse, L, 2)
    torch.cuda.synchronize()
    assert torch.equal(o, o_ref)
    assert torch.equal(ka.grad, dk) and torch.equal(va.grad, dv)
    assert rel_fro(f64(qa.grad), f64(dq)) < 1e-3  # dQ sums its reduce-adds in any order


def test_autograd_matches_oracle():
    q, k, v, do = random_attn_inputs(1, 2, 384, 64, "bf16", seed=32)
    L = torch.tensor([333], dtype=torch.int32)
    qa, ka, va = (t.cuda().requires_grad_(True) for t in (q, k, v))
    o = block_sparse_local_attention(qa, ka, va, L.cuda(), 1)
    (o.float() * do.cuda().float()).sum().backward()
    o_want, lse_want = attn_fwd_banded(f64(q), f64(k), f64(v), 1, [333])
    dq_w, dk_w, dv_w = attn_bwd_banded(f64(q), f64(k), f64(v), f64(do), 1, [333])
    assert max_abs(f64(o), o_want) < O_ATOL_BF16
    for got, want in ((qa.grad, dq_w), (ka.grad, dk_w), (va.grad, dv_w)):
        assert rel_fro(f64(got), want) < GRAD_RFRO_BF16


def test_collate_feeds_attention_end_to_end():
    """DNA strings -> IDs (collate) -> embeddings -> attention with the
    collator's lengths -> backward: padding rows get zero output and gradient."""
    torch.manual_seed(0)
    rng = np.random.default_rng(9)
    seqs = [rng.choice(np.frombuffer(b"ACGT", np.uint8), int(n)).tobytes() for n in (700, 1029, 90)]
    ids, lengths = collate(seqs, 6)
    heads, d = 2, 64
    emb = torch.nn.Embedding(4100, 3 * heads * d, device="cuda", dtype=torch.bfloat16)
    x = emb(ids)  # [batch, n_pad, 3 * heads * d]
    b, n = ids.shape
    q, k, v = (t.view(b, n, heads, d).transpose(1, 2) for t in x.split(heads * d, dim=-1))
    o = block_sparse_local_attention(q, k, v, lengths, 1)
    o.float().square().sum().backward()
    torch.cuda.synchronize()
    assert n == 1024 and lengths.cpu().tolist() == [695, 1024, 85]
    assert torch.isfinite(emb.weight.grad.float()).all()
    for row, L in enumerate(lengths.cpu().tolist()):
        assert (o[row, :, L:] == 0).all()


def test_autograd_causal_matches_direct_calls():
    q, k, v, do = (t.cuda() for t in random_attn_inputs(2, 2, 384, 64, "bf16", seed=41))
    L = torch.tensor([384, 250], dtype=torch.int32)
    qa, ka, va = (t.clone().requires_grad_(True) for t in (q, k, v))
    o = block_sparse_local_attention(qa, ka, va, L.cuda(), 2, causal=True)
    o.backward(do)
    o_ref, lse = run_fwd(q, k, v, L, 2, causal=True)
    dq, dk, dv = run_bwd(q, k, v, o_ref, do, lse, L, 2, causal=True)
    torch.cuda.synchronize()
    assert torch.equal(o, o_ref)
    assert torch.equal(ka.grad, dk) and torch.equal(va.grad, dv)
    assert rel_fro(f64(qa.grad), f64(dq)) < 1e-3
