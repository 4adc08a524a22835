"""Pins of the oracle's escape-coded streams (header flags bit 1) to facts that do
not come from the oracle itself.

An escape-coded block codes the exponents of a window of 2^w - 1 values at w
bits; code 2^w - 1 is the escape, and the escaped elements' exponent bytes follow
the codes as an exception list (the stream definition's section 12). The pages
give only the direction -- "ZipServ: Fast and Memory-Efficient LLM Inference
with Hardware-Aware Lossless Compression", Abstract: a fixed-length format that
decodes in constant time and in parallel -- so these pins hold the oracle to the
definition, by means that share nothing with its code:

- the choice of (w, base) against a brute force that counts every candidate
  window element by element, with the tie rules applied by sorting;
- every stream against a bit-serial reader written here (one bit at a time
  from the exponent plane, exceptions taken in element order), which rebuilds
  the input from the stream alone;
- block sizes, offsets and the total against per-block histograms in numpy;
- two streams worked out by hand (tests/golden/esc_*.txt) byte for byte;
- round trips on every BF16 bit pattern, edge sizes and every block size;
- rejection of streams that break the definition.
"""
import numpy as np
import pytest

import golden_io

BLOCKS = (128, 256, 512, 1024, 2048, 4096)


def exponents(words):
    return (np.asarray(words, dtype=np.int64) >> 7) & 0xFF


def brute_force_params(e):
    """(base, w, K) by enumerating every candidate; cost = ceil(L/8)*w + K,
    ties to the smaller w, then the larger base."""
    e = [int(v) for v in e]
    L = len(e)
    octets = -(-L // 8)
    cands = [(8 * octets, 8, 0, 0)]  # (cost, w, -base, K) of the raw block
    if all(v == e[0] for v in e):
        cands.append((0, 0, -e[0], 0))
    for w in range(1, 8):
        m = 2 ** w - 1
        for base in range(0, 256 - m):
            K = sum(1 for v in e if not (base <= v <= base + m - 1))
            cands.append((octets * w + K, w, -base, K))
    cost, w, nbase, K = min(cands)
    return -nbase, w, K


def words_from_exponents(rng, e):
    e = np.asarray(e, dtype=np.int64)
    return ((e << 7) | rng.integers(0, 128, e.size) | (rng.integers(0, 2, e.size) << 15)).astype(np.uint16)


def test_block_choice_by_brute_force(orc):
    rng = np.random.default_rng(11)
    cases = []
    for _ in range(400):
        L = int(rng.integers(1, 40))
        kind = int(rng.integers(0, 5))
        if kind == 0:    # a narrow cluster
            e = int(rng.integers(0, 250)) + rng.integers(0, 6, L)
        elif kind == 1:  # a cluster plus far outliers
            e = int(rng.integers(60, 200)) + rng.integers(0, 4, L)
            e[rng.integers(0, L, 1 + L // 10)] = rng.integers(0, 256, 1 + L // 10)
        elif kind == 2:  # anything
            e = rng.integers(0, 256, L)
        elif kind == 3:  # near the top: 255 can never sit in a window
            e = rng.integers(248, 256, L)
        else:            # geometric, like the exponents of Gaussian weights
            e = 125 - np.minimum(rng.geometric(0.5, L) - 1, 125)
        cases.append(np.clip(e, 0, 255))
    cases += [np.full(5, 7), np.full(9, 255), np.array([0, 255]), np.array([254, 255] * 4),
              np.array([0, 40, 80, 120, 160, 200, 240, 255])]
    for e in cases:
        words = words_from_exponents(rng, e)
        assert orc.esc_block_params(words) == brute_force_params(e), list(e)


# ----------------------------------------------------------------------------
# A bit-serial reader of escape-coded streams, written from the definition
# ----------------------------------------------------------------------------
def u64(stream, off):
    return int.from_bytes(bytes(stream[off:off + 8]), "little")


def read_escape_stream(stream, n, B):
    """Rebuild the BF16 words from the stream, one bit at a time."""
    A = lambda x: (x + 127) // 128 * 128
    nb = -(-n // B)
    off_offs = 128 + A(2 * nb)
    off_man = off_offs + A(4 * nb)
    off_exp = off_man + A(n)
    assert bytes(stream[0:4]) == b"WCB1"
    assert int.from_bytes(bytes(stream[12:16]), "little") == 2  # escape-coded
    assert [u64(stream, k) for k in (16, 24, 32, 40, 48, 56)] == [n, nb, 128, off_offs, off_man, off_exp]
    E = u64(stream, 64)
    assert u64(stream, 72) == off_exp + E == stream.size
    out = []
    for b in range(nb):
        L = min(B, n - b * B)
        base = int(stream[128 + 2 * b])
        w = int(stream[128 + 2 * b + 1])
        start = off_exp + 16 * int.from_bytes(bytes(stream[off_offs + 4 * b:off_offs + 4 * b + 4]), "little")
        code_bytes = -(-L // 8) * w
        nexc = 0
        for i in range(L):
            j, t = divmod(i, 8)
            c = 0
            for bit in range(w):  # element t of octet j: bits [t*w, t*w + w) of its w bytes
                pos = t * w + bit
                byte = int(stream[start + j * w + pos // 8])
                c |= ((byte >> (pos % 8)) & 1) << bit
            if w == 0:
                e = base
            elif w == 8:
                e = c
            elif c == 2 ** w - 1:
                e = int(stream[start + code_bytes + nexc])
                nexc += 1
            else:
                e = base + c
            s = int(stream[off_man + b * B + i])
            out.append(((s >> 7) << 15) | (e << 7) | (s & 0x7F))
        size = -(-(code_bytes + nexc) // 16) * 16
        assert not stream[start + code_bytes + nexc:start + size].any()  # zero padding
        nxt = (off_exp + 16 * int.from_bytes(bytes(stream[off_offs + 4 * b + 4:off_offs + 4 * b + 8]), "little")
               if b + 1 < nb else off_exp + E)
        assert nxt == start + size
    return np.array(out, dtype=np.uint16)


def numpy_sizes(words, B):
    """Per-block (w, base, K, padded size) from per-block exponent histograms."""
    n = words.size
    nb = -(-n // B)
    e = exponents(words)
    blk = np.arange(n) // B
    hist = np.zeros((nb, 256), np.int64)
    np.add.at(hist, (blk, e), 1)
    L = np.minimum(B, n - np.arange(nb) * B)
    octets = -(-L // 8)
    best = [(8 * octets[b], 8, 0, 0) for b in range(nb)]
    for b in range(nb):
        nz = np.nonzero(hist[b])[0]
        if nz.size == 1:
            best[b] = (0, 0, -int(nz[0]), 0)
    csum = np.concatenate([np.zeros((nb, 1), np.int64), np.cumsum(hist, axis=1)], axis=1)
    for w in range(1, 8):
        m = 2 ** w - 1
        inside = csum[:, m:256] - csum[:, 0:256 - m]  # windows [base, base + m - 1], base <= 255 - m
        cost = octets[:, None] * w + (L[:, None] - inside)
        for b in range(nb):
            c = cost[b]
            base = int(np.nonzero(c == c.min())[0].max())  # ties: the larger base
            cand = (int(c[base]), w, -base, int(L[b] - inside[b, base]))
            best[b] = min(best[b], cand)
    ws = np.array([x[1] for x in best], np.int64)
    bases = np.array([-x[2] for x in best], np.int64)
    K = np.array([x[3] for x in best], np.int64)
    sizes = -(-(octets * ws + K) // 16) * 16
    return ws, bases, K, sizes


def random_words(rng, n, kind):
    if kind == "gauss":
        f = (rng.standard_normal(n) * 0.02).astype(np.float32)
        return (f.view(np.uint32) >> 16).astype(np.uint16)
    if kind == "outliers":  # Gaussian with 1% of entries at 20 sigma and some zeros
        f = (rng.standard_normal(n) * 0.02).astype(np.float32)
        k = rng.random(n)
        f[k < 0.01] *= 1000.0
        f[k > 0.995] = 0.0
        return (f.view(np.uint32) >> 16).astype(np.uint16)
    if kind == "uniform":
        return rng.integers(0, 65536, n).astype(np.uint16)
    if kind == "zeros":
        return np.zeros(n, np.uint16)
    raise ValueError(kind)


SIZES = [0, 1, 7, 8, 9, 15, 16, 17, 127, 128, 129, 1000]


@pytest.mark.parametrize("B", BLOCKS)
@pytest.mark.parametrize("kind", ["gauss", "outliers", "uniform", "zeros"])
def test_escape_streams_against_reader_and_histograms(orc, B, kind):
    rng = np.random.default_rng(B + 7 * len(kind))
    sizes = SIZES + [B - 1, B, B + 1, 2 * B + 5]
    for n in sizes:
        words = random_words(rng, n, kind)
        stream = orc.compress_escape(words, B)
        assert stream.size <= orc.bound_escape(n, B)
        assert (orc.decompress_escape(stream, n, B) == words).all()
        nb = -(-n // B)
        if nb:
            ws, bases, K, sz = numpy_sizes(words, B)
            hdr = stream[128:128 + 2 * nb].view(np.uint16)
            assert ((hdr >> 8) == ws).all() and ((hdr & 0xFF) == bases).all()
            assert u64(stream, 64) == int(sz.sum())
        if n <= 2 * B + 5 and n <= 1200:  # the bit-serial reader is slow
            assert (read_escape_stream(stream, n, B) == words).all()


def test_bound_escape_is_the_padded_raw_size(orc):
    A = lambda x: (x + 127) // 128 * 128
    for B in BLOCKS:
        for n in [0, 1, 9, B, B + 3, 5 * B + 17]:
            nb = -(-n // B)
            L = np.minimum(B, n - np.arange(nb) * B)
            expect = 128 + A(2 * nb) + A(4 * nb) + A(n) + int((-(-((L + 7) // 8 * 8) // 16) * 16).sum())
            assert orc.bound_escape(n, B) == expect
    assert orc.bound_escape(1000, 100) == 0


@pytest.mark.parametrize("B", BLOCKS)
def test_all_65536_patterns(orc, B):
    words = np.random.default_rng(3).permutation(65536).astype(np.uint16)
    stream = orc.compress_escape(words, B)
    assert (orc.decompress_escape(stream, words.size, B) == words).all()
    natural = np.arange(65536, dtype=np.uint16)
    s2 = orc.compress_escape(natural, B)
    assert (orc.decompress_escape(s2, natural.size, B) == natural).all()
    if B == 128:  # every aligned run of 128 patterns shares one exponent: all w = 0
        assert not (s2[128:128 + 2 * 512].view(np.uint16) >> 8).any()
        assert u64(s2, 64) == 0


def test_gaussian_blocks_take_three_bits_and_beat_the_plain_width(orc):
    """Gaussian BF16 weights span 12-16 binades per block, but their exponent
    entropy is about 2.5 bits: the window code settles on w = 3 with a few
    percent of exceptions, and the stream is smaller than the plain one."""
    rng = np.random.default_rng(0)
    words = random_words(rng, 1 << 18, "gauss")
    for B in (512, 1024, 4096):
        s = orc.compress_escape(words, B)
        p = orc.compress(words, B)
        nb = words.size // B
        w = s[128:128 + 2 * nb].view(np.uint16) >> 8
        assert (w == 3).mean() > 0.99
        assert s.size < 0.95 * p.size
        e = exponents(words)
        counts = np.bincount(e, minlength=256) / e.size
        H = -(counts[counts > 0] * np.log2(counts[counts > 0])).sum()
        assert 2 * words.size / s.size < 16 / (8 + H)  # never better than the entropy bound


@pytest.mark.parametrize("name", golden_io.names("escape"))
def test_hand_derived_escape_streams(orc, name):
    B, words, expected, kind = golden_io.load_kind(name)
    assert kind == "escape"
    stream = orc.compress_escape(words, B)
    assert stream.size == expected.size
    assert (stream == expected).all(), np.nonzero(stream != expected)[0][:16]
    assert (orc.decompress_escape(expected, words.size, B) == words).all()
    assert (read_escape_stream(expected, words.size, B) == words).all()


def test_escape_decoder_rejects_corruption(orc):
    B, words, good, _ = golden_io.load_kind("esc_w2_two_escapes.txt")
    n = words.size
    assert orc.decompress_escape_status(good, n, B)[0] == orc.OK

    def status(mutate, nn=n, block=B):
        s = good.copy()
        s = mutate(s) if mutate else s
        return orc.decompress_escape_status(s, nn, block)[0]

    def setbyte(off, val):
        def f(s):
            s[off] = val
            return s
        return f

    assert status(setbyte(12, 0)) == orc.CORRUPT     # a plain stream's flags
    assert status(setbyte(12, 3)) == orc.CORRUPT     # FP32 and escape together
    assert status(setbyte(129, 9)) == orc.CORRUPT    # w = 9
    assert status(setbyte(128, 253)) == orc.CORRUPT  # base > 255 - (2^2 - 1)
    assert status(setbyte(516, 0x7e)) == orc.CORRUPT  # an exception inside the window
    assert status(setbyte(518, 1)) == orc.CORRUPT    # nonzero payload padding
    # sixteen escapes need 4 + 16 bytes: more than the block's 16-byte payload
    assert status(lambda s: (s.__setitem__(slice(512, 516), 0xFF), s)[1]) == orc.CORRUPT
    assert status(lambda s: s[:-1]) == orc.CORRUPT   # truncated
    assert status(None, nn=n - 1) == orc.CORRUPT
    assert status(None, block=256) == orc.CORRUPT
    # a plain stream is not an escape-coded one, and the other way round
    plain = orc.compress(words, B)
    assert orc.decompress_escape_status(plain, n, B)[0] == orc.CORRUPT
    assert orc.decompress_status(good, n, B)[0] == orc.CORRUPT
    # a nonzero code in a lane past the end of a block (13 elements: lanes 5..7
    # of octet 1 are unused; set the top bit of the octet, which is lane 7's)
    words13 = random_words(np.random.default_rng(9), 13, "gauss")
    s13 = orc.compress_escape(words13, 128)
    w = int(s13[129])
    assert 1 <= w <= 8 and orc.decompress_escape_status(s13, 13, 128)[0] == orc.OK
    off_exp = u64(s13, 56)
    s13[off_exp + 2 * w - 1] |= 0x80
    assert orc.decompress_escape_status(s13, 13, 128)[0] == orc.CORRUPT
