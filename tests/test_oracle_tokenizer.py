"""Pins for the tokenizer oracle, against values the NucleoByte page prints and
against Python's own base-4 / base-2 integer parsing (an independent route)."""

import numpy as np
import pytest

from oracle import kmer_ids, pack_2bit
from tests.conftest import read_golden

BASE4 = str.maketrans("ACGT", "0123")


def _golden_example():
    seq, idx, kmers = None, None, []
    for parts in read_golden("nucleobyte_mlm_example.txt"):
        if parts[0] == "sequence":
            seq = parts[1]
        elif parts[0] == "masked_index":
            idx = int(parts[1])
        elif parts[0] == "kmer":
            kmers.append((parts[1], int(parts[2])))
    return seq, idx, kmers


def test_page_printed_ids():
    """Each 6-mer the page prints decodes to the ID printed beside it."""
    _, _, kmers = _golden_example()
    assert len(kmers) == 3
    for kmer, page_id in kmers:
        assert kmer_ids(kmer.encode(), 6).tolist() == [page_id]


def test_page_sequence_all_windows_match_base4_parse():
    seq, _, _ = _golden_example()
    ids = kmer_ids(seq.encode(), 6)
    assert len(ids) == len(seq) - 5 == 25
    for p, got in enumerate(ids):
        assert int(got) == int(seq[p:p + 6].translate(BASE4), 4)
    # first and last windows, worked by hand: CCCAGG = 1*1024+1*256+1*64+0*16+2*4+2
    assert int(ids[0]) == 1354
    assert int(ids[24]) == 2425  # GCCTGC


def test_page_masked_index_is_garbled():
    """The window at the page's printed index 12 is TGGGAA (3744), one below the
    printed ground truth TGGGAC (3745), and TGGGAC occurs nowhere in the string:
    the page's position and its 6-mer disagree.  The ID<->6-mer mapping itself is
    pinned by test_page_printed_ids."""
    seq, idx, kmers = _golden_example()
    assert seq[idx:idx + 6] == "TGGGAA"
    assert int(kmer_ids(seq.encode(), 6)[idx]) == 3744
    assert kmers[0][0] not in seq


@pytest.mark.parametrize("k", [1, 2, 3, 4, 5, 6, 7])
def test_random_windows_match_base4_parse(k):
    rng = np.random.default_rng(100 + k)
    alphabet = np.frombuffer(b"ACGTN", dtype=np.uint8)
    s = alphabet[rng.integers(0, 5, size=200)].tobytes().decode()
    ids = kmer_ids(s.encode(), k)
    assert len(ids) == 200 - k + 1
    for p, got in enumerate(ids):
        w = s[p:p + k]
        want = 4 ** k if "N" in w else int(w.translate(BASE4), 4)
        assert int(got) == want


def test_invalid_bytes_flag_window():
    s = b"ACGTACGTNACGTACGTa\nCGTAC"
    ids = kmer_ids(s, 6)
    for p in range(len(s) - 5):
        w = s[p:p + 6]
        if all(c in b"ACGT" for c in w):
            assert ids[p] == int(w.decode().translate(BASE4), 4)
        else:
            assert ids[p] == 4096


def test_short_inputs():
    assert kmer_ids(b"", 6).shape == (0,)
    assert kmer_ids(b"ACGTA", 6).shape == (0,)
    assert kmer_ids(b"ACGTAC", 6).tolist() == [int("012301", 4)]
    assert pack_2bit(b"").shape == (0,)


def test_pack_known_bytes():
    assert pack_2bit(b"ACGT").tolist() == [0x1B]
    assert pack_2bit(b"TTTT").tolist() == [0xFF]
    assert pack_2bit(b"AAAA").tolist() == [0x00]
    assert pack_2bit(b"ACG").tolist() == [0b00011000]  # tail slot zero
    assert pack_2bit(b"N").tolist() == [0]
    assert pack_2bit(b"ACGTG").tolist() == [0x1B, 0x80]


def test_pack_random_matches_bitstring_parse():
    rng = np.random.default_rng(7)
    alphabet = np.frombuffer(b"ACGTN", dtype=np.uint8)
    for n in [1, 2, 3, 4, 5, 17, 64, 131]:
        s = alphabet[rng.integers(0, 5, size=n)].tobytes().decode()
        bits = "".join("00" if c == "N" else format("ACGT".index(c), "02b") for c in s)
        bits += "0" * (-len(bits) % 8)
        want = [int(bits[i:i + 8], 2) for i in range(0, len(bits), 8)]
        assert pack_2bit(s.encode()).tolist() == want


# ---------------------------------------------------------------- model IDs

def test_model_ids_reproduce_the_page_masked_position():
    """With padding at 0 and window IDs shifted up by one, the model ID at the
    page's masked position 12 is the ID the page prints there (3745)."""
    from oracle.tokenizer import model_ids_batch

    seq, idx, kmers = _golden_example()
    ids, lengths = model_ids_batch([seq.encode()], 6)
    assert int(ids[0, idx]) == kmers[0][1] == 3745
    # every window: its base-4 value plus one; then padding up to the ceiling 32
    assert lengths.tolist() == [25] and ids.shape == (1, 32)
    for p in range(25):
        assert int(ids[0, p]) == int(seq[p:p + 6].translate(BASE4), 4) + 1
    assert ids[0, 25:].tolist() == [0] * 7


def test_model_ids_flag_pad_and_vocabulary():
    from oracle.tokenizer import model_ids_batch

    ids, lengths = model_ids_batch([b"ACGTNACGTAC", b"ACGTA", b"", b"TTTTTTT"], 6)
    assert lengths.tolist() == [6, 0, 0, 2]
    assert ids.shape == (4, 32)
    # windows 0..5 of ACGTNACGTAC: those holding the N (byte 4) are 4^6 + 1
    assert ids[0, :6].tolist() == [4097] * 5 + [int("ACGTAC".translate(BASE4), 4) + 1]
    assert ids[3, :2].tolist() == [4096, 4096]  # TTTTTT = 4095 raw
    assert ids[1].tolist() == [0] * 32 and ids[2].tolist() == [0] * 32
    assert int(ids.max()) < 4100  # the page's vocab_size


@pytest.mark.parametrize("windows,ceiling", [(0, 0), (1, 32), (31, 32), (32, 32), (33, 64),
                                             (4091, 4096), (4096, 4096)])
def test_dynamic_ceiling(windows, ceiling):
    from oracle.tokenizer import ceiling as ceil32

    assert ceil32(windows) == ceiling


def test_model_ids_truncate_to_explicit_pad():
    from oracle.tokenizer import model_ids_batch

    ids, lengths = model_ids_batch([b"ACGTACGTACGT"], 3, n_pad=4)
    assert lengths.tolist() == [4]
    assert ids[0].tolist() == [int(w.translate(BASE4), 4) + 1 for w in ("ACG", "CGT", "GTA", "TAC")]
