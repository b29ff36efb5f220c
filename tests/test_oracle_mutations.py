"""Plant plausible mistakes in a private copy of the oracle (on the CPU) and
check that independent pins reject every one of them."""

import importlib.util
import math
import os

import numpy as np
import pytest
from scipy.special import softmax

import oracle.attention as att
import oracle.tokenizer as tok

SRC_ATT = open(att.__file__).read()
SRC_TOK = open(tok.__file__).read()


def _load_mutant(src, name):
    spec = importlib.util.spec_from_loader(name, loader=None)
    mod = importlib.util.module_from_spec(spec)
    exec(compile(src, name, "exec"), mod.__dict__)
    return mod


def _fwd_pin_fails(mod):
    """Softmax over the visible keys enumerated by hand, with a length mask."""
    rng = np.random.default_rng(0)
    n, d, R, L = 128, 8, 1, 90
    q, k, v = (rng.standard_normal((1, 1, n, d)) for _ in range(3))
    o, lse = mod.attn_fwd_dense(q, k, v, R, lengths=[L])
    o_b, _ = mod.attn_fwd_banded(q, k, v, R, lengths=[L])
    for i in range(L):
        ib = i // 32
        keys = [j for j in range(L) if abs(j // 32 - ib) <= R]
        s = np.array([q[0, 0, i] @ k[0, 0, j] for j in keys]) / math.sqrt(d)
        want = softmax(s) @ v[0, 0, keys]
        if not (np.allclose(o[0, 0, i], want, atol=1e-10) and np.allclose(o_b[0, 0, i], want, atol=1e-10)):
            return True
    return False


def _bwd_pin_fails(mod):
    """Central differences of sum(O * dO) on a tiny case, for both oracles."""
    rng = np.random.default_rng(1)
    n, d, R, L = 64, 4, 0, 50
    q, k, v, do = (rng.standard_normal((1, 1, n, d)) for _ in range(4))
    h = 1e-6

    def loss(qq, kk, vv):
        o, _ = att.attn_fwd_dense(qq, kk, vv, R, lengths=[L])  # the unmutated forward
        return float((o * do).sum())

    for fn in (mod.attn_bwd_dense, mod.attn_bwd_banded):
        grads = fn(q, k, v, do, R, lengths=[L])
        for which, g in enumerate(grads):
            for (i, t) in [(3, 1), (40, 2), (33, 0), (49, 3)]:
                p = [q.copy(), k.copy(), v.copy()]
                m = [q.copy(), k.copy(), v.copy()]
                p[which][0, 0, i, t] += h
                m[which][0, 0, i, t] -= h
                fd = (loss(*p) - loss(*m)) / (2 * h)
                if abs(fd - g[0, 0, i, t]) > 1e-6 * (1 + abs(fd)):
                    return True
    return False


ATT_MUTATIONS = [
    ("band off by one", "blk[None, :]) <= R\n", "blk[None, :]) < R\n"),
    ("band j1 off by one", "min(nb - 1, i + R)", "min(nb - 1, i + R - 1)"),
    ("scale dropped", "scale = 1.0 / math.sqrt(d)", "scale = 1.0"),
    ("keys past length kept", "k0, k1 = j0 * BLOCK, min((j1 + 1) * BLOCK, L)  # keys past L are masked",
     "k0, k1 = j0 * BLOCK, (j1 + 1) * BLOCK"),
    ("length mask dropped", "m &= (np.arange(n) < length)[None, :]", "pass"),
    ("D sign", "dS = P * (dP - D[:, None])  # softmax gradient", "dS = P * (dP + D[:, None])  # softmax gradient"),
    ("D sign banded", "dS = P * (dP - D[:, None])\n", "dS = P * (dP + D[:, None])\n"),
    ("D dropped", "dS = P * (dP - D[:, None])  # softmax gradient", "dS = P * dP  # softmax gradient"),
    ("dK transposed", "dk[b, h] = scale * (dS.T @ q[b, h])", "dk[b, h] = scale * (dS @ q[b, h])"),
    ("dV without P^T", "dv[b, h] = P.T @ dO", "dv[b, h] = P @ dO"),
    ("dQ scale dropped", "dq[b, h] = scale * (dS @ k[b, h])", "dq[b, h] = dS @ k[b, h]"),
    ("banded dK scale dropped", "dk[b, h, k0:k1] += scale * (dS.T @ Qi)", "dk[b, h, k0:k1] += dS.T @ Qi"),
    ("softmax not normalised", "E / np.where(l > 0, l, 1.0)[:, None]", "E"),
]


@pytest.mark.parametrize("name,old,new", ATT_MUTATIONS, ids=[m[0] for m in ATT_MUTATIONS])
def test_attention_mutation_is_caught(name, old, new):
    assert old in SRC_ATT, name
    mod = _load_mutant(SRC_ATT.replace(old, new), "mutant_" + name.replace(" ", "_"))
    assert _fwd_pin_fails(mod) or _bwd_pin_fails(mod), name


TOK_MUTATIONS = [
    ("code order", 'zip(b"ACGT", range(4))', 'zip(b"ACTG", range(4))'),
    ("LSB first", "4 ** (k - 1 - t)", "4 ** t"),
    ("flag value", "ids[bad] = N_FLAG_BASE ** k", "ids[bad] = 0"),
    ("pack order", "(quads[:, 0] << 6) | (quads[:, 1] << 4) | (quads[:, 2] << 2) | quads[:, 3]",
     "(quads[:, 3] << 6) | (quads[:, 2] << 4) | (quads[:, 1] << 2) | quads[:, 0]"),
]


@pytest.mark.parametrize("name,old,new", TOK_MUTATIONS, ids=[m[0] for m in TOK_MUTATIONS])
def test_tokenizer_mutation_is_caught(name, old, new):
    assert old in SRC_TOK, name
    mod = _load_mutant(SRC_TOK.replace(old, new), "mutant_tok")
    page = {"TGGGAC": 3745, "TGAAGT": 3595, "GGCCCC": 2645}
    ok = all(mod.kmer_ids(s.encode(), 6).tolist() == [v] for s, v in page.items())
    ok &= mod.kmer_ids(b"ACGTNA", 6).tolist() == [4096]
    ok &= mod.pack_2bit(b"ACGTG").tolist() == [0x1B, 0x80]
    assert not ok, name


MODEL_ID_MUTATIONS = [
    ("no id shift", "ids[b, :m] = r[:m].astype(np.int64) + 1", "ids[b, :m] = r[:m].astype(np.int64)"),
    ("pad id", "PAD_ID = 0", "PAD_ID = 4099"),
    ("ceiling rounds down", "return -(-max(int(n_windows_max), 0) // block) * block",
     "return (max(int(n_windows_max), 0) // block) * block"),
]


@pytest.mark.parametrize("name,old,new", MODEL_ID_MUTATIONS, ids=[m[0] for m in MODEL_ID_MUTATIONS])
def test_model_id_mutation_is_caught(name, old, new):
    assert old in SRC_TOK, name
    mod = _load_mutant(SRC_TOK.replace(old, new), "mutant_tok_ids")
    page_seq = b"CCCAGGGTCCGATGGGAAAGTGTAGCCTGC"
    ids, lengths = mod.model_ids_batch([page_seq, b"ACG"], 6)
    ok = ids.shape == (2, 32) and int(ids[0, 12]) == 3745 and lengths.tolist() == [25, 0]
    ok = ok and ids[0, 25:].tolist() == [0] * 7 and ids[1].tolist() == [0] * 32
    assert not ok, name


def _causal_pin_fails(mod):
    """Causal band: keys enumerated by hand per row, both oracles, fwd; and
    central differences of the causal loss for the banded backward."""
    rng = np.random.default_rng(5)
    n, d, R, L = 96, 4, 1, 80
    q, k, v, do = (rng.standard_normal((1, 1, n, d)) for _ in range(4))
    o, _ = mod.attn_fwd_dense(q, k, v, R, lengths=[L], causal=True)
    o_b, _ = mod.attn_fwd_banded(q, k, v, R, lengths=[L], causal=True)
    for i in range(L):
        keys = [j for j in range(L) if 0 <= i // 32 - j // 32 <= R and j <= i]
        s = np.array([q[0, 0, i] @ k[0, 0, j] for j in keys]) / math.sqrt(d)
        want = softmax(s) @ v[0, 0, keys]
        if not (np.allclose(o[0, 0, i], want, atol=1e-10) and np.allclose(o_b[0, 0, i], want, atol=1e-10)):
            return True
    h = 1e-6

    def loss(kk):
        oo, _ = att.attn_fwd_dense(q, kk, v, R, lengths=[L], causal=True)  # the unmutated forward
        return float((oo * do).sum())

    _, dk, _ = mod.attn_bwd_banded(q, k, v, do, R, lengths=[L], causal=True)
    for i in (5, 31, 32, 63, 64, 79):
        p, m = k.copy(), k.copy()
        p[0, 0, i, 1] += h
        m[0, 0, i, 1] -= h
        if abs((loss(p) - loss(m)) / (2 * h) - dk[0, 0, i, 1]) > 1e-6:
            return True
    return False


CAUSAL_MUTATIONS = [
    ("causal mask off by one", "m &= np.arange(n)[None, :] <= np.arange(n)[:, None]",
     "m &= np.arange(n)[None, :] < np.arange(n)[:, None]"),
    ("causal cut off by one", "return np.where(ki <= qi, S, -np.inf)", "return np.where(ki < qi, S, -np.inf)"),
    # (keeping block i + 1 would be harmless: the triangle masks it whole)
    ("causal band drops the diagonal block", "(i if causal else", "(i - 1 if causal else"),
    ("causal cut skipped in backward", "                if causal:\n                    S = _causal_cut(S, r0, k0)\n                P, _, _",
     "                P, _, _"),
]


@pytest.mark.filterwarnings("ignore::RuntimeWarning")  # the mutants' own arithmetic
@pytest.mark.parametrize("name,old,new", CAUSAL_MUTATIONS, ids=[m[0] for m in CAUSAL_MUTATIONS])
def test_causal_mutation_is_caught(name, old, new):
    assert old in SRC_ATT, name
    mod = _load_mutant(SRC_ATT.replace(old, new), "mutant_causal")
    try:
        caught = _causal_pin_fails(mod)
    except ValueError:  # the mutant cannot even evaluate the pins (an empty band)
        caught = True
    assert caught, name


def _saved_pin_fails(mod):
    """The backward from saved outputs: equal to the unmutated plain backward
    when O and lse come from the forward, and a row's lse raised by ln 2
    halves that row's P (so its dV contribution)."""
    rng = np.random.default_rng(7)
    for causal in (False, True):
        q, k, v, do = (rng.standard_normal((1, 2, 128, 4)) for _ in range(4))
        o, lse = att.attn_fwd_banded(q, k, v, 1, [100], causal=causal)
        want = att.attn_bwd_banded(q, k, v, do, 1, [100], causal=causal)
        got = mod.attn_bwd_from_saved(q, k, v, o, do, lse, 1, [100], causal=causal)
        if not all(np.allclose(g, w, atol=1e-10) for g, w in zip(got, want)):
            return True
    q, k, v, do = (rng.standard_normal((1, 1, 64, 4)) for _ in range(4))
    o, lse = att.attn_fwd_banded(q, k, v, 0)
    do[0, 0, 32:] = 0
    lse2 = lse.copy()
    lse2[0, 0, :32] += math.log(2.0)
    dv1 = mod.attn_bwd_from_saved(q, k, v, o, do, lse, 0)[2]
    dv2 = mod.attn_bwd_from_saved(q, k, v, o, do, lse2, 0)[2]
    return not np.allclose(dv2, dv1 / 2, atol=1e-12)


SAVED_MUTATIONS = [
    ("saved backward renormalises instead of using lse",
     "P = np.where(np.isfinite(li), np.exp(S - li), 0.0)",
     "P = np.where(np.isfinite(li), _softmax_rows(S)[0], 0.0)"),
    ("saved backward row term from dO only", "D = (dOi * o[b, h, r0:r0 + rows]).sum(axis=1)",
     "D = (dOi * dOi).sum(axis=1)"),
    ("saved backward drops the scale of lse", "np.exp(S - li)", "np.exp(S / scale - li)"),
]


@pytest.mark.filterwarnings("ignore::RuntimeWarning")
@pytest.mark.parametrize("name,old,new", SAVED_MUTATIONS, ids=[m[0] for m in SAVED_MUTATIONS])
def test_saved_backward_mutation_is_caught(name, old, new):
    assert SRC_ATT.count(old) == 1, name
    mod = _load_mutant(SRC_ATT.replace(old, new), "mutant_saved")
    assert _saved_pin_fails(mod), name
