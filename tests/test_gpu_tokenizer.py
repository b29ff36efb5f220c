"""GPU parity of nb_tokenize_kmer against the tokenizer oracle: bit-exact."""

import numpy as np
import pytest
import torch

import block_sparse_local_nb_b200 as nb
from block_sparse_local_nb_b200.inputs import DNA_BYTES, make_dna
from oracle import kmer_ids, pack_2bit
from tests.conftest import read_golden

pytestmark = pytest.mark.gpu


def _run(seq_np: np.ndarray, k=6, seq_off=0, ids_off=0, packed_off=0, want_ids=True,
         want_packed=True):
    """Tokenize on the GPU with optional byte offsets applied to each buffer."""
    n = seq_np.shape[0]
    raw = torch.zeros(n + seq_off + 64, dtype=torch.uint8, device="cuda")
    if n:
        raw[seq_off:seq_off + n] = torch.from_numpy(seq_np.copy()).cuda()
    nwin = max(0, n - k + 1)
    # 2-byte elements (uint16 viewed as int16), guard value 0xBEEF
    ids_raw = torch.full((nwin + ids_off + 16,), 0xBEEF - 0x10000, dtype=torch.int16, device="cuda")
    packed_raw = torch.full(((n + 3) // 4 + packed_off + 16,), 0xAB, dtype=torch.uint8,
                            device="cuda")
    ids_ptr = ids_raw.data_ptr() + 2 * ids_off if want_ids else None
    packed_ptr = packed_raw.data_ptr() + packed_off if want_packed else None
    nb.nb_tokenize_kmer(raw.data_ptr() + seq_off, n, ids_ptr, packed_ptr, k)
    torch.cuda.synchronize()
    ids = ids_raw[ids_off:ids_off + nwin].cpu().numpy().view(np.uint16)
    packed = packed_raw[packed_off:packed_off + (n + 3) // 4].cpu().numpy()
    # guard bytes after the outputs must be untouched
    tail_ids = ids_raw[ids_off + nwin:ids_off + nwin + 8].cpu().numpy().view(np.uint16)
    tail_packed = packed_raw[packed_off + (n + 3) // 4:].cpu().numpy()
    if want_ids:
        assert (tail_ids == 0xBEEF).all()
    if want_packed:
        assert (tail_packed == 0xAB).all()
    return ids, packed


def test_page_example_bit_exact():
    seq = next(p[1] for p in read_golden("nucleobyte_mlm_example.txt") if p[0] == "sequence")
    s = np.frombuffer(seq.encode(), dtype=np.uint8)
    ids, packed = _run(s)
    np.testing.assert_array_equal(ids, kmer_ids(s, 6))
    np.testing.assert_array_equal(packed, pack_2bit(s))


@pytest.mark.parametrize("n", [0, 1, 3, 5, 6, 7, 15, 16, 17, 21, 22, 23, 24, 25, 31, 32, 33, 47,
                               64, 100, 255, 256, 257, 1000, 4099, 65536 + 13])
def test_lengths_bit_exact(n):
    s = make_dna(n, seed=1000 + n, n_prob=0.05)
    ids, packed = _run(s)
    np.testing.assert_array_equal(ids, kmer_ids(s, 6))
    np.testing.assert_array_equal(packed, pack_2bit(s))


@pytest.mark.parametrize("k", [1, 2, 3, 4, 5, 7])
def test_other_k_bit_exact(k):
    s = make_dna(3001, seed=k, n_prob=0.02)
    ids, packed = _run(s, k=k)
    np.testing.assert_array_equal(ids, kmer_ids(s, k))
    np.testing.assert_array_equal(packed, pack_2bit(s))


@pytest.mark.parametrize("seq_off,ids_off,packed_off", [(1, 0, 0), (3, 1, 1), (8, 3, 2),
                                                        (15, 7, 3), (0, 5, 0)])
def test_unaligned_buffers(seq_off, ids_off, packed_off):
    s = make_dna(5000 + seq_off, seed=77, n_prob=0.01)
    ids, packed = _run(s, seq_off=seq_off, ids_off=ids_off, packed_off=packed_off)
    np.testing.assert_array_equal(ids, kmer_ids(s, 6))
    np.testing.assert_array_equal(packed, pack_2bit(s))


def test_other_bytes_are_invalid():
    s = np.frombuffer(b"ACGTacgtNRYKM\n\r ACGTACGTTTGCA" * 9 + bytes(range(256)), dtype=np.uint8)
    ids, packed = _run(s)
    np.testing.assert_array_equal(ids, kmer_ids(s, 6))
    np.testing.assert_array_equal(packed, pack_2bit(s))


def test_single_output():
    s = make_dna(777, seed=3)
    ids, _ = _run(s, want_packed=False)
    np.testing.assert_array_equal(ids, kmer_ids(s, 6))
    _, packed = _run(s, want_ids=False)
    np.testing.assert_array_equal(packed, pack_2bit(s))


def test_full_size_2p28_bit_exact():
    """The 2**28-byte workload (1% N), whole output compared with the oracle."""
    s = make_dna(DNA_BYTES)
    seq = torch.from_numpy(s).cuda()
    ids = torch.empty(DNA_BYTES - 5, dtype=torch.int16, device="cuda")
    packed = torch.empty(DNA_BYTES // 4, dtype=torch.uint8, device="cuda")
    nb.nb_tokenize_kmer(seq, DNA_BYTES, ids, packed, 6)
    torch.cuda.synchronize()
    got_ids = ids.cpu().numpy().view(np.uint16)
    np.testing.assert_array_equal(got_ids, kmer_ids(s, 6))
    np.testing.assert_array_equal(packed.cpu().numpy(), pack_2bit(s))


# ------------------------------------------------------- batch to model IDs

def _run_batch(seqs, k=6, n_pad=None, lead=3):
    """nb_tokenize_batch on `seqs` concatenated after `lead` bytes (so sequences
    start at arbitrary byte offsets); returns (ids, lengths) and checks that the
    guard row after the output and the guard entry after the lengths are untouched."""
    from oracle.tokenizer import ceiling

    offsets = [lead]
    for s in seqs:
        offsets.append(offsets[-1] + len(s))
    # bases before the first and after the last sequence must not be read into them
    blob = b"ACGT" * 4 + b"Z" * lead + b"".join(seqs) + b"ACGT" * 4
    offsets = [o + 16 for o in offsets]
    dev = torch.frombuffer(bytearray(blob), dtype=torch.uint8).cuda()
    off = torch.tensor(offsets, dtype=torch.int64, device="cuda")
    if n_pad is None:
        n_pad = ceiling(max([max(len(s) - k + 1, 0) for s in seqs], default=0))
    ids = torch.full((len(seqs) + 1, max(n_pad, 1)), -7, dtype=torch.int64, device="cuda")
    lengths = torch.full((len(seqs) + 1,), -7, dtype=torch.int32, device="cuda")
    nb.nb_tokenize_batch(dev, off, len(seqs), k, ids, lengths, n_pad)
    torch.cuda.synchronize()
    assert (ids[len(seqs)] == -7).all() and int(lengths[len(seqs)]) == -7
    return ids[:len(seqs), :n_pad].cpu().numpy(), lengths[:len(seqs)].cpu().numpy()


def test_batch_page_example():
    from oracle.tokenizer import model_ids_batch

    seq = [p for p in read_golden("nucleobyte_mlm_example.txt") if p[0] == "sequence"][0][1]
    ids, lengths = _run_batch([seq.encode()])
    want, want_len = model_ids_batch([seq.encode()], 6)
    assert np.array_equal(ids, want) and np.array_equal(lengths, want_len)
    assert int(ids[0, 12]) == 3745


@pytest.mark.parametrize("k", [1, 3, 6, 7])
def test_batch_random_matches_oracle(k):
    from oracle.tokenizer import model_ids_batch

    rng = np.random.default_rng(40 + k)
    alphabet = np.frombuffer(b"ACGTACGTACGTNacgt\n", dtype=np.uint8)
    lens = [0, 1, k - 1, k, k + 1, 31 + k, 32 + k, 33 + k] + rng.integers(0, 3000, 40).tolist()
    seqs = [alphabet[rng.integers(0, alphabet.size, int(n))].tobytes() for n in lens]
    ids, lengths = _run_batch(seqs, k, lead=k)
    want, want_len = model_ids_batch(seqs, k)
    assert np.array_equal(lengths, want_len)
    assert np.array_equal(ids, want)


def test_batch_truncates_to_n_pad():
    from oracle.tokenizer import model_ids_batch

    rng = np.random.default_rng(3)
    seqs = [rng.choice(np.frombuffer(b"ACGT", np.uint8), n).tobytes() for n in (10, 100, 300)]
    ids, lengths = _run_batch(seqs, 6, n_pad=64)
    want, want_len = model_ids_batch(seqs, 6, n_pad=64)
    assert lengths.tolist() == [5, 64, 64] == want_len.tolist()
    assert np.array_equal(ids, want)


def test_batch_training_sized():
    """1024 sequences of up to 4101 bases (the training batches' shape)."""
    from oracle.tokenizer import model_ids_batch

    rng = np.random.default_rng(11)
    alphabet = np.frombuffer(b"ACGTACGTACGTACGTACGTACGTACGTACGTACGTACGTACGTACGTACGTACGTACGTACGTACGTACGTACGTACGTACGTACGTACGTACGTN",
                             np.uint8)
    seqs = [alphabet[rng.integers(0, alphabet.size, int(n))].tobytes()
            for n in rng.integers(1024, 4102, 1024)]
    ids, lengths = _run_batch(seqs, 6)
    want, want_len = model_ids_batch(seqs, 6)
    assert ids.shape == (1024, 4096)
    assert np.array_equal(lengths, want_len) and np.array_equal(ids, want)
