"""Oracle for the fused 2-bit DNA k-mer tokenizer.

TEST INFRASTRUCTURE ONLY (see the package docstring).

Following the NucleoByte page: section 1 ("Token Blur": a hard-coded,
bit-packed sliding window over the bases), section 2 item 1 ("Fused 2-Bit
Tokenization": bases packed into integer IDs), section 5 ("Architecture Size":
k = 6, a 4096-entry k-mer vocabulary plus padding/mask; "Evaluation Output
Verification": 'TGGGAC' = 3745, 'TGAAGT' = 3595, 'GGCCCC' = 2645).

Definition written out here:

* Each base gets a 2-bit code A=0, C=1, G=2, T=3 (the three printed IDs decode
  exactly under this code with the first base most significant).  Every other
  byte value (N, lower case, IUPAC letters, newlines) is "invalid".
* Window p (0 <= p <= len - k) has ID sum_{t<k} code[p+t] * 4**(k-1-t); a window
  that contains an invalid byte gets the flag ID 4**k (4096 for k = 6).
* The packed base stream holds 4 bases per byte, the first base in bits 7..6;
  an invalid base is stored as 0 (a 2-bit code cannot hold it; the ID stream
  carries the flag); unused slots of the final byte are 0.

Model input IDs of a batch (section 2 item 2 "Dynamic Ceiling Hardware
Alignment": a batch is padded up to the nearest multiple of the block size 32;
section 5: a 4096-entry vocabulary "plus padding/mask"; section 6: vocab_size
4100 and input IDs drawn from 1 upward).  Reading: ID 0 is padding and every
raw window ID is shifted up by one, so a window of valid bases has ID raw + 1
in 1..4**k, a window with an invalid byte 4**k + 1, and the mask ID is
4**k + 2.  The page's MLM example supports the shift: its masked position 12
holds the window TGGGAA (raw 3744) and the page prints ID 3745 there.
"""

from __future__ import annotations

import numpy as np

N_FLAG_BASE = 4  # the flag ID of a window with an invalid byte is N_FLAG_BASE ** k


def _codes(seq) -> tuple[np.ndarray, np.ndarray]:
    """Return (code, valid) for a byte sequence: code in 0..3 (0 where invalid)."""
    s = np.frombuffer(seq, dtype=np.uint8) if isinstance(seq, (bytes, bytearray)) else np.asarray(seq, dtype=np.uint8)
    lut = np.full(256, -1, dtype=np.int16)
    for letter, c in zip(b"ACGT", range(4)):
        lut[letter] = c
    raw = lut[s]
    valid = raw >= 0
    code = np.where(valid, raw, 0).astype(np.uint16)
    return code, valid


def kmer_ids(seq, k: int = 6) -> np.ndarray:
    """Sliding-window k-mer IDs (uint16, one per window, stride 1)."""
    if not 1 <= k <= 7:
        raise ValueError("k must be in 1..7 so that the flag ID fits uint16")
    code, valid = _codes(seq)
    n = code.shape[0]
    nwin = n - k + 1
    if nwin <= 0:
        return np.zeros(0, dtype=np.uint16)
    ids = np.zeros(nwin, dtype=np.uint16)
    bad = np.zeros(nwin, dtype=bool)
    for t in range(k):  # sum of shifted slices: code[p+t] * 4**(k-1-t)
        ids += code[t:t + nwin] * np.uint16(4 ** (k - 1 - t))
        bad |= ~valid[t:t + nwin]
    ids[bad] = N_FLAG_BASE ** k
    return ids


def pack_2bit(seq) -> np.ndarray:
    """Packed 2-bit base stream: ceil(len/4) bytes, first base in the top bits."""
    code, _ = _codes(seq)
    n = code.shape[0]
    nbytes = (n + 3) // 4
    padded = np.zeros(nbytes * 4, dtype=np.uint16)
    padded[:n] = code
    quads = padded.reshape(nbytes, 4)
    out = (quads[:, 0] << 6) | (quads[:, 1] << 4) | (quads[:, 2] << 2) | quads[:, 3]
    return out.astype(np.uint8)


PAD_ID = 0


def ceiling(n_windows_max: int, block: int = 32) -> int:
    """The dynamic ceiling: the smallest multiple of `block` holding n_windows_max."""
    return -(-max(int(n_windows_max), 0) // block) * block


def model_ids_batch(seqs, k: int = 6, n_pad: int | None = None):
    """Model input IDs (int64 [batch, n_pad]) and window counts (int32 [batch]).

    Row b holds kmer_ids(seqs[b]) + 1 (the flag window becomes 4**k + 1), then
    PAD_ID; n_pad defaults to the ceiling of the longest row.  Rows longer than
    n_pad keep their first n_pad windows.
    """
    raw = [kmer_ids(s, k) for s in seqs]
    counts = [r.shape[0] for r in raw]
    if n_pad is None:
        n_pad = ceiling(max(counts, default=0))
    ids = np.full((len(seqs), n_pad), PAD_ID, dtype=np.int64)
    lengths = np.zeros(len(seqs), dtype=np.int32)
    for b, r in enumerate(raw):
        m = min(r.shape[0], n_pad)
        ids[b, :m] = r[:m].astype(np.int64) + 1
        lengths[b] = m
    return ids, lengths
