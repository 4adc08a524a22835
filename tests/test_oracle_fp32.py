"""Pins for the oracle's FP32 streams (CPU only).

An FP32 stream codes the high 16-bit halves of the words exactly as a BF16
stream and keeps the low halves raw in a plane between the mantissa and the
exponent planes (flags bit 0 set, the plane's offset at header byte 80). The
pins: round trips; the FP32 exponent field seen through float arithmetic; the
closed-form size; the stream rebuilt independently by splicing the (separately
pinned) BF16 oracle's stream of the high halves with a numpy-built low plane;
and rejection of the ways an FP32 stream can be malformed.
"""
import numpy as np
import pytest

pytestmark = pytest.mark.filterwarnings("ignore::RuntimeWarning")

BLOCKS = [128, 256, 512, 1024, 2048, 4096]


def A(x):
    return (x + 127) // 128 * 128


def fp32_words(rng, n, kind):
    if kind == "gauss":
        return (rng.standard_normal(n).astype(np.float32) * 0.02).view(np.uint32)
    if kind == "random":
        return rng.integers(0, 2 ** 32, n, dtype=np.uint64).astype(np.uint32)
    if kind == "specials":
        pool = np.array([0x00000000, 0x80000000, 0x00000001, 0x807FFFFF, 0x7F800000, 0xFF800000,
                         0x7FC00000, 0x7FC00001, 0x7F800001, 0xFFFFFFFF, 0x3F800000, 0x00400000],
                        dtype=np.uint32)
        return pool[rng.integers(0, pool.size, n)]
    raise ValueError(kind)


@pytest.mark.parametrize("B", BLOCKS)
@pytest.mark.parametrize("kind", ["gauss", "random", "specials"])
def test_fp32_round_trip(orc, B, kind):
    rng = np.random.default_rng(B + len(kind))
    for n in (0, 1, 7, 8, 9, B - 1, B, B + 1, 3 * B + 5, 20000):
        x = fp32_words(rng, n, kind)
        s = orc.compress_f32(x, B)
        assert np.array_equal(orc.decompress_f32(s, n, B), x), (n, kind)


def test_fp32_high_half_exponent_is_the_float_exponent(orc):
    """The e-field of a word's high half is the biased FP32 exponent (frexp)."""
    rng = np.random.default_rng(7)
    x = (rng.standard_normal(5000) * np.exp(rng.uniform(-60, 60, 5000))).astype(np.float32)
    x = x[np.isfinite(x) & (x != 0) & (np.abs(x) >= np.finfo(np.float32).tiny)]
    words = x.view(np.uint32)
    _, ex = np.frexp(x.astype(np.float64))
    for w, e in zip(words[:2000], ex[:2000]):
        assert orc.exponent(int(w >> 16)) == int(e) + 126


def widths(hi, B):
    e = ((hi.astype(np.int64) >> 7) & 0xFF)
    ws = []
    for b in range(0, hi.size, B):
        blk = e[b:b + B]
        ws.append(int(blk.max() - blk.min()).bit_length())
    return ws


@pytest.mark.parametrize("B", [128, 1024, 4096])
def test_fp32_closed_form_size(orc, B):
    rng = np.random.default_rng(B)
    for n in (1, 100, B, 5 * B + 3, 30000):
        x = fp32_words(rng, n, "gauss")
        hi = (x >> 16).astype(np.uint16)
        nb = -(-n // B)
        E = sum(-(-min(B, n - b * B) // 8) * w for b, w in zip(range(nb), widths(hi, B)))
        total = 128 + A(2 * nb) + A(4 * nb) + A(n) + A(2 * n) + E
        s = orc.compress_f32(x, B)
        assert s.size == total
        assert orc.bound_f32(n, B) == orc.bound(n, B) + A(2 * n)


@pytest.mark.parametrize("B", [256, 1024])
def test_fp32_stream_is_the_bf16_stream_of_the_high_halves_plus_a_low_plane(orc, B):
    rng = np.random.default_rng(11 + B)
    for n in (0, 5, 1000, 9000):
        x = fp32_words(rng, n, "gauss")
        hi = (x >> 16).astype(np.uint16)
        lo = (x & 0xFFFF).astype(np.uint16)
        b16 = orc.compress(hi, B)
        nb = -(-n // B)
        off_man = 128 + A(2 * nb) + A(4 * nb)
        off_low = off_man + A(n)
        off_exp16 = off_man + A(n)
        off_exp = off_low + A(2 * n)
        E = int(b16[64:72].view(np.uint64)[0])
        want = np.zeros(off_exp + E, dtype=np.uint8)
        want[:off_low] = b16[:off_low]                      # header, headers, offsets, mantissas
        want[off_low:off_low + 2 * n] = lo.view(np.uint8)   # the low plane
        want[off_exp:] = b16[off_exp16:off_exp16 + E]       # exponent plane
        want[12:16] = np.frombuffer(np.uint32(1).tobytes(), np.uint8)           # flags
        want[56:64] = np.frombuffer(np.uint64(off_exp).tobytes(), np.uint8)     # off_exp
        want[72:80] = np.frombuffer(np.uint64(off_exp + E).tobytes(), np.uint8)  # total
        want[80:88] = np.frombuffer(np.uint64(off_low).tobytes(), np.uint8)     # off_low
        assert np.array_equal(orc.compress_f32(x, B), want), n


def test_fp32_malformed_streams_are_rejected(orc):
    rng = np.random.default_rng(13)
    n, B = 3000, 512
    x = fp32_words(rng, n, "gauss")
    s = orc.compress_f32(x, B)
    assert orc.decompress_f32_status(s, n, B)[0] == 0
    # an FP32 stream is not a BF16 stream, nor the other way round
    assert orc.decompress_status(s, n, B)[0] == orc.CORRUPT
    b16 = orc.compress((x >> 16).astype(np.uint16), B)
    assert orc.decompress_f32_status(b16, n, B)[0] == orc.CORRUPT
    nb = -(-n // B)
    off_low = 128 + A(2 * nb) + A(4 * nb) + A(n)
    for pos, val in ((80, 0), (81, 1), (100, 1), (off_low + 2 * n, 1), (off_low - 1, 1)):
        bad = s.copy()
        bad[pos] = val if bad[pos] != val else val ^ 1
        assert orc.decompress_f32_status(bad, n, B)[0] == orc.CORRUPT, pos
    assert orc.decompress_f32_status(s[:-1], n, B)[0] == orc.CORRUPT


def test_fp16_words_need_at_most_three_more_bits_than_their_exponent(orc):
    """FP16 words through the 16-bit path: a block's width is at most bits(d) + 3,
    d the span of the 5-bit FP16 exponents (taken from float arithmetic)."""
    rng = np.random.default_rng(17)
    B = 256
    for scale in (1e-3, 0.02, 1.0, 300.0):
        h = (rng.standard_normal(B * 40) * scale).astype(np.float16)
        h = np.where(np.abs(h) < np.float16(6.2e-5), np.float16(6.2e-5), h)  # normals only
        words = h.view(np.uint16)
        _, ex = np.frexp(h.astype(np.float64))
        for b in range(40):
            blk, eb = words[b * B:(b + 1) * B], ex[b * B:(b + 1) * B]
            d = int(eb.max() - eb.min())
            base, w = orc.block_params(blk)
            assert w <= d.bit_length() + 3
        s = orc.compress(words, B)
        assert np.array_equal(orc.decompress(s, words.size, B), words)
