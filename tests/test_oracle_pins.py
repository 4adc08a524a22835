"""Pins of the CPU oracle to facts that do not come from the oracle itself.

- The split is checked against the binary structure of BF16 numbers, computed
  with floating-point arithmetic (numpy frexp / isnan / signbit), not bit masks.
- The width rule is checked by brute force over every (base, w) pair.
- The hierarchical halving pack is checked against a bit-by-bit construction
  of the closed form sum_t v_t * 2^(t*w), exhaustively for w <= 2.
- Stream sizes, block headers and offsets are recomputed by vectorised numpy
  from the closed form 128 + A(2nb) + A(4nb) + A(n) + sum_b ceil(L_b/8)*w_b.
- Three streams worked out by hand (tests/golden/) must match byte for byte.
- Round trip identity on every BF16 bit pattern and on edge sizes.

The method: "ENEC: A Lossless AI Model Compression Method Enabling Fast
Inference on Ascend NPUs", Abstract (per-block fixed-length code, bit-width
quantization, hierarchical halving bit-packing, branch-free remap, prefix sum).
"""
import itertools

import numpy as np
import pytest

import golden_io

pytestmark = pytest.mark.filterwarnings("ignore:invalid value encountered in cast")

BLOCKS = (128, 256, 512, 1024, 2048, 4096)


def bf16_as_f32(words):
    return (np.asarray(words, dtype=np.uint32) << 16).view(np.float32)


# ----------------------------------------------------------------------------
# Step 1: split / merge
# ----------------------------------------------------------------------------
def test_split_matches_bf16_number_structure(orc):
    x = np.arange(65536, dtype=np.uint16)
    e = np.array([orc.exponent(int(v)) for v in x], dtype=np.int64)
    s = np.array([orc.signman(int(v)) for v in x], dtype=np.int64)
    f = bf16_as_f32(x)
    # sign bit of s is the number's sign (also for -0 and NaN)
    assert ((s >> 7) == np.signbit(f)).all()
    finite = np.isfinite(f)
    assert (e[~finite] == 255).all() and (e[finite] < 255).all()
    a = np.abs(f.astype(np.float64))
    normal = finite & (a >= 2.0 ** -126)
    frac, ex = np.frexp(a[normal])  # a = frac * 2^ex, frac in [0.5, 1)
    assert (e[normal] == ex - 1 + 127).all()  # a = 2^(e-127) * (1 + m/128)
    assert ((s[normal] & 0x7F) == np.round((2 * frac - 1) * 128)).all()
    sub = finite & ~normal  # zero and denormals: a = m * 2^-133, e = 0
    assert (e[sub] == 0).all()
    assert ((s[sub] & 0x7F) == np.round(a[sub] * 2.0 ** 133)).all()
    assert ((s[np.isinf(f)] & 0x7F) == 0).all()
    assert ((s[np.isnan(f)] & 0x7F) != 0).all()


def test_merge_is_the_inverse_of_split(orc):
    for x in range(65536):
        assert orc.merge(orc.exponent(x), orc.signman(x)) == x
    # and split o merge is the identity on all (e, s) pairs: a bijection
    seen = set()
    for e in range(256):
        for s in range(256):
            x = orc.merge(e, s)
            assert (orc.exponent(x), orc.signman(x)) == (e, s)
            seen.add(x)
    assert len(seen) == 65536


# ----------------------------------------------------------------------------
# Step 2: width quantization
# ----------------------------------------------------------------------------
def test_bits_is_binary_length(orc):
    for d in list(range(300)) + [2**20 - 1, 2**20, 2**31 - 1]:
        assert orc.bits(d) == d.bit_length()


def test_width_rule_by_brute_force(orc):
    """Every (base, w) that represents the block is enumerated; the oracle must
    pick the smallest w, with base = the block's minimum exponent (0 when raw)."""
    rng = np.random.default_rng(1)
    bases = np.arange(256)[None, :, None]
    widths = np.arange(9)[:, None, None]
    for _ in range(2000):
        L = int(rng.integers(1, 24))
        span = int(rng.choice([0, 1, 2, 3, 7, 8, 15, 16, 40, 127, 128, 200, 255]))
        lo0 = int(rng.integers(0, 256 - span))
        e = lo0 + rng.integers(0, span + 1, L)
        words = ((e << 7) | rng.integers(0, 128, L) | (rng.integers(0, 2, L) << 15)).astype(np.uint16)
        base, w = orc.block_params(words)
        ok = ((e[None, None, :] - bases) >= 0) & ((e[None, None, :] - bases) < (1 << widths))
        valid = ok.all(axis=2)  # [w, base]
        wmin = int(np.argmax(valid.any(axis=1)))
        assert w == wmin
        assert valid[w, base]
        if w < 8:
            assert base == e.min()
        else:
            assert base == 0


# ----------------------------------------------------------------------------
# Step 4: hierarchical halving pack
# ----------------------------------------------------------------------------
def bit_serial_octet(values, w):
    """The closed form sum_t v_t * 2^(t*w), built one bit at a time."""
    o = 0
    for t, v in enumerate(values):
        for bit in range(w):
            if (v >> bit) & 1:
                o |= 1 << (t * w + bit)
    return o


def test_pack_one_value_in_each_lane(orc):
    for w in range(9):
        for t in range(8):
            for v in range(1 << w):
                vals = [0] * 8
                vals[t] = v
                assert orc.pack_octet(vals, w) == v * 2 ** (t * w)


@pytest.mark.parametrize("w", [1, 2])
def test_pack_every_octet_small_widths(orc, w):
    for vals in itertools.product(range(1 << w), repeat=8):
        o = orc.pack_octet(list(vals), w)
        assert o == bit_serial_octet(vals, w)
        assert orc.unpack_octet(o, w) == list(vals)


def test_pack_random_octets_all_widths(orc):
    rng = np.random.default_rng(2)
    for w in range(9):
        for _ in range(3000):
            vals = [int(v) for v in rng.integers(0, 1 << w, 8)]
            o = orc.pack_octet(vals, w)
            assert o == bit_serial_octet(vals, w)
            assert o < 2 ** (8 * w)
            assert orc.unpack_octet(o, w) == vals


# ----------------------------------------------------------------------------
# Whole streams: closed-form layout recomputed with numpy
# ----------------------------------------------------------------------------
def A(x):
    return (x + 127) // 128 * 128


def numpy_layout(words, B):
    """Block headers, offsets and section offsets from vectorised numpy."""
    n = words.size
    nb = -(-n // B)
    f = bf16_as_f32(words)
    # exponent from the number itself: 255 for Inf/NaN, 0 for zero/denormal
    a = np.abs(f.astype(np.float64))
    e = np.where(~np.isfinite(f), 255,
                 np.where(a >= 2.0 ** -126, np.frexp(np.where(a > 0, a, 1.0))[1] - 1 + 127, 0))
    starts = np.arange(nb) * B
    L = np.minimum(B, n - starts)
    lo = np.minimum.reduceat(e, starts) if nb else np.zeros(0, np.int64)
    hi = np.maximum.reduceat(e, starts) if nb else np.zeros(0, np.int64)
    w = np.frexp((hi - lo).astype(np.float64))[1].astype(np.int64)  # bit length
    base = np.where(w == 8, 0, lo)
    sizes = (L + 7) // 8 * w
    offs = np.concatenate([[0], np.cumsum(sizes)[:-1]]) if nb else np.zeros(0, np.int64)
    E = int(sizes.sum())
    off_offs = 128 + A(2 * nb)
    off_man = off_offs + A(4 * nb)
    off_exp = off_man + A(n)
    return dict(nb=nb, base=base, w=w, offs=offs, E=E, off_offs=off_offs, off_man=off_man,
                off_exp=off_exp, total=off_exp + E)


def u64(stream, off):
    return int(stream[off:off + 8].view(np.uint64)[0])


def check_stream_against_numpy(stream, words, B):
    exp = numpy_layout(words, B)
    n, nb = words.size, exp["nb"]
    assert stream.size == exp["total"]
    assert int(stream[0:4].view(np.uint32)[0]) == 0x31424357
    assert bytes(stream[0:4]) == b"WCB1"
    assert u64(stream, 16) == n and u64(stream, 24) == nb
    assert [u64(stream, k) for k in (32, 40, 48, 56, 64, 72)] == [
        128, exp["off_offs"], exp["off_man"], exp["off_exp"], exp["E"], exp["total"]]
    hdr = stream[128:128 + 2 * nb].view(np.uint16)
    assert ((hdr & 0xFF) == exp["base"]).all() and ((hdr >> 8) == exp["w"]).all()
    offs = stream[exp["off_offs"]:exp["off_offs"] + 4 * nb].view(np.uint32).astype(np.int64)
    assert (offs * 16 == exp["offs"]).all()
    # mantissa plane: the sign and the 7 stored fraction bits of each number
    f = bf16_as_f32(words)
    man = stream[exp["off_man"]:exp["off_man"] + n].astype(np.int64)
    assert ((man >> 7) == np.signbit(f)).all()
    assert ((man & 0x7F) == (words & 0x7F)).all()
    # zero padding between sections and in the header tail
    for a_, b_ in ((80, 128), (128 + 2 * nb, exp["off_offs"]),
                   (exp["off_offs"] + 4 * nb, exp["off_man"]), (exp["off_man"] + n, exp["off_exp"])):
        assert not stream[a_:b_].any()


def random_words(rng, n, kind):
    if kind == "gauss":
        f = (rng.standard_normal(n) * 0.02).astype(np.float32)
        return (f.view(np.uint32) >> 16).astype(np.uint16)
    if kind == "uniform":
        return rng.integers(0, 65536, n).astype(np.uint16)
    if kind == "zeros":
        return np.zeros(n, np.uint16)
    if kind == "narrow":  # exponents within a few binades
        return ((rng.integers(120, 124, n) << 7) | rng.integers(0, 65536, n) & 0x807F).astype(np.uint16)
    raise ValueError(kind)


SIZES = [0, 1, 7, 8, 9, 15, 16, 17, 127, 128, 129, 1000]


@pytest.mark.parametrize("B", BLOCKS)
@pytest.mark.parametrize("kind", ["gauss", "uniform", "zeros", "narrow"])
def test_stream_layout_and_round_trip(orc, B, kind):
    rng = np.random.default_rng(B + len(kind))
    for n in SIZES + [B - 1, B, B + 1, 3 * B + 5, 7 * B + 100]:
        words = random_words(rng, n, kind)
        stream = orc.compress(words, B)
        check_stream_against_numpy(stream, words, B)
        assert stream.size <= orc.bound(n, B)
        assert (orc.decompress(stream, n, B) == words).all()


def test_bound_is_the_all_raw_size(orc):
    for B in BLOCKS:
        for n in [0, 1, 9, B, B + 3, 5 * B + 17]:
            nb = -(-n // B)
            L = np.minimum(B, n - np.arange(nb) * B)
            expect = 128 + A(2 * nb) + A(4 * nb) + A(n) + int(((L + 7) // 8 * 8).sum())
            assert orc.bound(n, B) == expect
    for bad in (0, 64, 100, 384, 8192, 2**31):
        assert orc.bound(1000, bad) == 0


# ----------------------------------------------------------------------------
# Exhaustive BF16 patterns and special cases
# ----------------------------------------------------------------------------
def test_all_65536_patterns_natural_order(orc):
    words = np.arange(65536, dtype=np.uint16)
    # at B=128 every 128-aligned run shares bits 15..7, hence one exponent: all w = 0
    stream = orc.compress(words, 128)
    check_stream_against_numpy(stream, words, 128)
    nb = 512
    assert not (stream[128:128 + 2 * nb].view(np.uint16) >> 8).any()
    assert u64(stream, 64) == 0
    assert (orc.decompress(stream, words.size, 128) == words).all()
    for B in BLOCKS[1:]:
        s = orc.compress(words, B)
        check_stream_against_numpy(s, words, B)
        assert (orc.decompress(s, words.size, B) == words).all()


@pytest.mark.parametrize("B", BLOCKS)
def test_all_65536_patterns_permuted(orc, B):
    words = np.random.default_rng(3).permutation(65536).astype(np.uint16)
    stream = orc.compress(words, B)
    check_stream_against_numpy(stream, words, B)
    assert (orc.decompress(stream, words.size, B) == words).all()


def test_all_zero_tensor(orc):
    n, B = 10_000, 512
    stream = orc.compress(np.zeros(n, np.uint16), B)
    nb = -(-n // B)
    assert stream.size == 128 + A(2 * nb) + A(4 * nb) + A(n)
    assert not (stream[128:128 + 2 * nb].view(np.uint16)).any()  # base 0, w 0


def test_uniform_random_takes_raw_path(orc):
    rng = np.random.default_rng(4)
    words = rng.integers(0, 65536, 64 * 128).astype(np.uint16)
    stream = orc.compress(words, 128)
    lay = numpy_layout(words, 128)
    w = stream[128:128 + 2 * 64].view(np.uint16) >> 8
    assert (w == 8).sum() == (lay["w"] == 8).sum() == 64


def test_constant_exponent_block_has_no_payload(orc):
    rng = np.random.default_rng(5)
    words = ((121 << 7) | (rng.integers(0, 65536, 4096) & 0x807F)).astype(np.uint16)
    stream = orc.compress(words, 1024)
    assert u64(stream, 64) == 0
    assert (stream[128:136].view(np.uint16) == 121).all()


def test_empty_tensor(orc):
    stream = orc.compress(np.zeros(0, np.uint16), 256)
    assert stream.size == 128
    assert [u64(stream, k) for k in (16, 24, 32, 40, 48, 56, 64, 72)] == [0, 0, 128, 128, 128, 128, 0, 128]
    assert orc.decompress(stream, 0, 256).size == 0


# ----------------------------------------------------------------------------
# Hand-derived streams
# ----------------------------------------------------------------------------
@pytest.mark.parametrize("name", golden_io.names())
def test_hand_derived_streams(orc, name):
    B, words, expected = golden_io.load(name)
    stream = orc.compress(words, B)
    assert stream.size == expected.size
    assert (stream == expected).all(), np.nonzero(stream != expected)[0][:16]
    assert (orc.decompress(expected, words.size, B) == words).all()


# ----------------------------------------------------------------------------
# The oracle decoder rejects streams that break the definition
# ----------------------------------------------------------------------------
def test_decoder_rejects_corruption(orc):
    rng = np.random.default_rng(6)
    words = random_words(rng, 3 * 256 + 40, "gauss")
    B = 256
    good = orc.compress(words, B)
    assert orc.decompress_status(good, words.size, B)[0] == orc.OK
    lay = numpy_layout(words, B)

    def bad(mutate, n=words.size, block=B):
        s = good.copy()
        s = mutate(s) if mutate else s
        return orc.decompress_status(s, n, block)[0]

    def setbyte(off, val):
        def f(s):
            s[off] = val
            return s
        return f

    assert bad(setbyte(0, 0x58)) == orc.CORRUPT                # magic
    assert bad(setbyte(4, 2)) == orc.CORRUPT                   # version
    assert bad(setbyte(129, 9)) == orc.CORRUPT                 # w = 9
    assert bad(setbyte(lay["off_offs"] + 4, 0xFF)) == orc.CORRUPT  # offset of block 1
    assert bad(lambda s: s[:-1]) == orc.CORRUPT                # truncated
    assert bad(lambda s: s[:100]) == orc.CORRUPT               # shorter than the header
    assert bad(None, n=words.size - 1) == orc.CORRUPT          # n disagrees
    assert bad(None, block=512) == orc.CORRUPT                 # B disagrees
    assert bad(setbyte(lay["off_man"] + words.size, 1)) == orc.CORRUPT  # padding
