"""Pins of the oracle's tANS-coded streams (the exponents entropy-coded by tabled
asymmetric numeral systems, 32 interleaved lane streams per chunk; "MINE:
Entropy-coded Memory-efficient Inference for Large Language Models", Abstract,
names a tANS-family GPU coder, dtANS-LLM, with hyper-parameters trading ratio
against decoding cost; the format is this project's reading).

Independent of the oracle's own code:
- two streams worked out by hand (tests/golden/tans_*.txt);
- a decoder written here from the format definition, bit by bit, that must
  rebuild the input from the oracle's streams (word order, refill rule, state
  transitions, mantissa merge);
- the defining property of a tANS table: for each exponent e, the ranges
  [next[X], next[X] + 2^nb[X]) of the states X that decode e tile [0, L)
  exactly once, and e owns f[e] states;
- the normalization's sum, support and closeness to the histogram;
- the coded size against the exponent's empirical entropy (a lossless code
  cannot beat it; tANS with 2^R states comes within a small overhead);
- round trips of all 65,536 patterns and edge sizes, and rejection of
  corrupted streams.
"""
import numpy as np
import pytest

import golden_io
from test_oracle_pins import bf16_as_f32  # noqa: F401  (keeps the pin modules together)

CHUNKS = (1024, 2048, 4096, 8192)


def gauss_words(rng, n, std=0.02):
    f = (rng.standard_normal(n) * std).astype(np.float32)
    return (f.view(np.uint32) >> 16).astype(np.uint16)


def A(x):
    return (x + 127) // 128 * 128


def py_decode(stream, n, C):
    """The format definition, read directly: header, counts, spread table,
    per-chunk 32 lane states and the shared word stream."""
    st = np.asarray(stream, dtype=np.uint8)
    le = lambda off, k: int.from_bytes(st[off:off + k].tobytes(), "little")  # noqa: E731
    assert le(0, 4) == 0x31424357 and le(12, 4) == 4 and le(16, 8) == n and le(8, 4) == C
    R = le(88, 4)
    L = 1 << R
    nb = -(-n // C)
    off_offs = 128 + 512
    off_man = off_offs + A(4 * nb)
    off_exp = off_man + A(n)
    E = le(64, 8)
    freq = [le(128 + 2 * e, 2) for e in range(256)]
    # the spread: exponents in order, f[e] states each, stepping by L/2 + L/8 + 3
    sym = [0] * L
    p = 0
    for e in range(256):
        for _ in range(freq[e]):
            sym[p] = e
            p = (p + (L >> 1) + (L >> 3) + 3) % L
    count = list(freq)
    nbits, nxt = [0] * L, [0] * L
    for X in range(L):
        v = count[sym[X]]
        count[sym[X]] += 1
        nbits[X] = R - (v.bit_length() - 1)
        nxt[X] = (v << nbits[X]) - L
    out = np.zeros(n, np.uint16)
    consumed = 0
    for c in range(nb):
        start = 16 * le(off_offs + 4 * c, 4)
        end = 16 * le(off_offs + 4 * c + 4, 4) if c + 1 < nb else E
        pay = off_exp + start
        ln = min(C, n - c * C)
        X = [le(pay + 2 * l, 2) for l in range(32)]
        bits = [0] * 32      # the lane's buffered bits, as an integer
        held = [0] * 32
        w = 0
        for k in range(-(-ln // 32)):
            for l in range(32):
                if l + 32 * k < ln and held[l] < R:
                    bits[l] |= le(pay + 64 + 4 * w, 4) << held[l]
                    held[l] += 32
                    w += 1
            for l in range(32):
                i = l + 32 * k
                if i >= ln:
                    continue
                s = X[l]
                e = sym[s]
                take = nbits[s]
                X[l] = nxt[s] + (bits[l] & ((1 << take) - 1))
                consumed += take
                bits[l] >>= take
                held[l] -= take
                m = int(st[off_man + c * C + i])
                out[c * C + i] = ((m & 0x80) << 8) | (e << 7) | (m & 0x7F)
        assert all(x == 0 for x in X)  # every lane ends in state 0
        assert 64 + 4 * w <= end - start
    py_decode.consumed = consumed
    return out


@pytest.mark.parametrize("name", ["tans_one_symbol.txt", "tans_two_symbols.txt"])
def test_hand_derived_streams(orc, name):
    C, R, words, expected = golden_io.load_tans(name)
    got = orc.compress_tans(words, C, R)
    assert got.size == expected.size
    assert np.array_equal(got, expected)
    assert np.array_equal(orc.decompress_tans(expected, words.size, C), words)
    assert np.array_equal(py_decode(expected, words.size, C), words)


@pytest.mark.parametrize("C,R", [(1024, 8), (1024, 12), (2048, 11), (4096, 9), (8192, 10)])
def test_independent_decoder_rebuilds_the_input(orc, C, R):
    rng = np.random.default_rng(C + R)
    n = 2 * C + 77
    w = gauss_words(rng, n)
    w[rng.integers(0, n, 40)] = rng.integers(0, 65536, 40)  # rare exponents: tiny counts
    s = orc.compress_tans(w, C, R)
    assert np.array_equal(py_decode(s, n, C), w)


@pytest.mark.parametrize("R", [8, 9, 10, 11, 12])
def test_table_ranges_tile_the_states(orc, R):
    """For each exponent the next-state ranges of its states partition [0, L)."""
    rng = np.random.default_rng(R)
    L = 1 << R
    counts = np.zeros(256, np.uint64)
    counts[rng.integers(100, 160, 30)] = rng.integers(1, 100000, 30)
    counts[7] = 1  # a symbol far below 1/L of the total
    f = orc.tans_normalize(counts, R)
    sym, nb, nxt = orc.tans_table(f, R)
    for e in np.flatnonzero(f):
        states = np.flatnonzero(sym == e)
        assert states.size == f[e]
        cover = np.zeros(L, np.int64)
        for X in states:
            cover[int(nxt[X]):int(nxt[X]) + (1 << int(nb[X]))] += 1
        assert (cover == 1).all(), e


@pytest.mark.parametrize("R", [8, 11, 12])
def test_normalization(orc, R):
    rng = np.random.default_rng(100 + R)
    L = 1 << R
    for trial in range(50):
        counts = np.zeros(256, np.uint64)
        k = int(rng.integers(1, 256))
        idx = rng.choice(256, k, replace=False)
        counts[idx] = rng.integers(1, 10 ** int(rng.integers(1, 7)), k)
        f = orc.tans_normalize(counts, R).astype(np.int64)
        assert f.sum() == L
        assert np.array_equal(f > 0, counts > 0)           # support kept
        ideal = counts.astype(np.float64) * L / counts.sum()
        # off by less than one except the one entry that absorbs the rounding
        off = np.abs(f - ideal)
        assert (np.sort(off)[:-1] < 1.0 + 1e-9).all()
    f = orc.tans_normalize(np.eye(256, dtype=np.uint64)[9] * 5, R)
    assert f[9] == L and f.sum() == L


def test_bits_read_against_the_table_entropy(orc):
    """A tANS code spends log2(L / f[e]) bits on exponent e, up to the states'
    information: the bits the decoder reads total n times the cross-entropy of
    the histogram under the normalized counts, within R bits per lane (the first
    state carries R bits, and the last is 0); and that cross-entropy lies just
    above the empirical entropy."""
    rng = np.random.default_rng(7)
    n, C, R = 1 << 16, 4096, 11
    w = gauss_words(rng, n)
    e = (w >> 7) & 0xFF
    counts = np.bincount(e, minlength=256)
    p = counts / n
    H = float(-(p[p > 0] * np.log2(p[p > 0])).sum())
    f = orc.tans_normalize(counts.astype(np.uint64), R).astype(np.float64)
    Hf = float(-(p[p > 0] * np.log2(f[p > 0] / (1 << R))).sum())
    assert H <= Hf < H + 0.01
    s = orc.compress_tans(w, C, R)
    assert np.array_equal(py_decode(s, n, C), w)
    lanes = 32 * (n // C)
    assert abs(py_decode.consumed - n * Hf) <= lanes * R


def test_size_against_the_exponent_entropy(orc):
    """Exponent bits per element: above the empirical entropy less the states'
    information, below it plus the per-chunk states (32 x 16 bits) and at most
    two words per lane beyond its bits (a partly filled last word, and a refill
    the rule takes by the count held)."""
    rng = np.random.default_rng(7)
    n = 1 << 20
    w = gauss_words(rng, n)
    e = (w >> 7) & 0xFF
    p = np.bincount(e, minlength=256) / n
    H = float(-(p[p > 0] * np.log2(p[p > 0])).sum())
    for C in (4096, 8192):
        s = orc.compress_tans(w, C, 11)
        off_exp = 128 + 512 + A(4 * (-(-n // C))) + A(n)
        bits = 8.0 * (s.size - off_exp) / n
        assert H - 0.01 < bits < H + (512.0 + 2048.0) / C + 0.02, (C, bits, H)


@pytest.mark.parametrize("C", CHUNKS)
def test_round_trip_every_pattern(orc, C):
    rng = np.random.default_rng(C)
    allw = np.arange(65536, dtype=np.uint16)
    for w in (allw, rng.permutation(allw)):
        for R in (8, 12):
            s = orc.compress_tans(w, C, R)
            assert np.array_equal(orc.decompress_tans(s, w.size, C), w)


@pytest.mark.parametrize("n", [0, 1, 31, 32, 33, 1023, 1024, 1025, 5000, 8193])
def test_round_trip_edge_sizes(orc, n):
    rng = np.random.default_rng(n)
    w = gauss_words(rng, n)
    for C in CHUNKS:
        s = orc.compress_tans(w, C, 11)
        assert np.array_equal(orc.decompress_tans(s, n, C), w)
        assert s.size <= orc.bound_tans(n, C, 11)


def test_rejects_corruption(orc):
    rng = np.random.default_rng(11)
    n, C = 3000, 1024
    w = gauss_words(rng, n)
    s = orc.compress_tans(w, C, 10)
    nb = -(-n // C)
    off_exp = 128 + 512 + A(4 * nb) + A(n)
    cases = []
    b = s.copy(); b[12] = 5; cases.append(b)                    # flags
    b = s.copy(); b[88] = 13; cases.append(b)                   # table log out of range
    b = s.copy(); b[128 + 2 * 120] ^= 1; cases.append(b)        # counts no longer sum to L
    b = s.copy(); b[off_exp] ^= 0x04; cases.append(b)           # a lane's first state
    b = s.copy(); b[off_exp + 1] = 0xFF; cases.append(b)        # a state >= L
    b = s.copy(); b[off_exp + 70] ^= 0x10; cases.append(b)      # a word's bit
    b = s.copy(); b[128 + 512] = 1; cases.append(b)             # chunk offset
    for k, b in enumerate(cases):
        rc, _ = orc.decompress_tans_status(b, n, C)
        assert rc == 3, k
    rc, _ = orc.decompress_tans_status(s[:-16], n, C)           # truncated
    assert rc == 3
    assert orc.decompress_tans_status(s, n, C)[0] == 0
