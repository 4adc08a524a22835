"""GPU parity of escape-coded streams (header flags bit 1) against the CPU oracle.

An escape-coded block codes a window of 2^w - 1 exponents at w bits and lists
the exponents of the elements outside it after its codes; the stream
definition's section 12 fixes every byte. As for plain streams the bar is
bit-exactness: wc_compress_escape's stream equals the oracle's byte for byte
and wc_decompress_escape gives back the input words bit for bit, on the
hand-derived streams, at ragged edge sizes for every block size, on every BF16
bit pattern, on the workloads (outliers, all-zero rows, random slabs,
denormals, NaN payloads) and in batches. Corrupt streams must end in
WC_ERR_CORRUPT_STREAM without harming the device. All calls go through the
C-ABI library.
"""
import numpy as np
import pytest
import torch

import golden_io
from gpu_util import to_gpu_words, words_np

pytestmark = pytest.mark.gpu

BLOCKS = (128, 256, 512, 1024, 2048, 4096)


def random_words(rng, n, kind):
    if kind == "gauss":
        f = (rng.standard_normal(n) * 0.02).astype(np.float32)
        return (f.view(np.uint32) >> 16).astype(np.uint16)
    if kind == "outliers":  # heavy tails and zeros: many escapes per block
        f = (rng.standard_normal(n) * 0.02).astype(np.float32)
        k = rng.random(n)
        f[k < 0.02] *= 1000.0
        f[k > 0.99] = 0.0
        return (f.view(np.uint32) >> 16).astype(np.uint16)
    if kind == "uniform":
        return rng.integers(0, 65536, n).astype(np.uint16)
    if kind == "zeros":
        return np.zeros(n, np.uint16)
    if kind == "mixed":  # gaussian with specials (255 is always an exception) and random slabs
        w = random_words(rng, n, "gauss")
        if n:
            pos = rng.integers(0, n, max(1, n // 50))
            w[pos] = rng.choice([0x0000, 0x8000, 0x7F80, 0xFF80, 0x7FC0, 0xFFFF, 0x0001, 0x807F], pos.size)
            a = int(rng.integers(0, n))
            w[a:a + 300] = rng.integers(0, 65536, len(w[a:a + 300]))
        return w
    raise ValueError(kind)


def gpu_compress_escape(wc, words_t, B):
    c = wc.compress_escape(words_t, B)
    torch.cuda.synchronize()
    assert c.status.item() == 0
    return c.stream().cpu().numpy()


def gpu_decompress_escape(wc, stream, n, B, device, stream_bytes=None):
    s = torch.from_numpy(np.ascontiguousarray(stream)).to(device)
    status = torch.zeros(1, dtype=torch.int32, device=device)
    out = torch.empty(n, dtype=torch.int16, device=device)
    wc.decompress_escape(s, n, B, out=out, status=status,
                         nbytes=stream.size if stream_bytes is None else stream_bytes)
    torch.cuda.synchronize()
    return out.cpu().numpy().view(np.uint16), int(status.item())


def roundtrip_vs_oracle(orc, wc, words, B, device):
    ref = orc.compress_escape(words, B)
    got = gpu_compress_escape(wc, to_gpu_words(words, device), B)
    assert got.size == ref.size, (got.size, ref.size)
    diff = np.nonzero(got != ref)[0]
    assert diff.size == 0, "first differing bytes at %s" % diff[:8]
    dec, status = gpu_decompress_escape(wc, ref, words.size, B, device)
    assert status == 0
    assert np.array_equal(dec, words)


@pytest.mark.parametrize("name", golden_io.names("escape"))
def test_hand_derived_escape_streams(wclib, cuda, name):
    B, words, expected, _ = golden_io.load_kind(name)
    got = gpu_compress_escape(wclib, to_gpu_words(words, cuda), B)
    assert np.array_equal(got, expected)
    dec, status = gpu_decompress_escape(wclib, expected, words.size, B, cuda)
    assert status == 0 and np.array_equal(dec, words)


SIZES = [1, 7, 8, 9, 15, 16, 17, 127, 128, 129, 1000, 4095, 4096, 4097, 8191, 8192, 8193,
         3 * 8192 + 5, 100_003, 1 << 20]
KINDS = ["gauss", "outliers", "uniform", "zeros", "mixed"]


@pytest.mark.parametrize("B", BLOCKS)
@pytest.mark.parametrize("kind", KINDS)
def test_edge_sizes_vs_oracle(orc, wclib, cuda, B, kind):
    rng = np.random.default_rng(20 * B + KINDS.index(kind))
    for n in SIZES + [B - 1, B + 1, 5 * B + 3]:
        roundtrip_vs_oracle(orc, wclib, random_words(rng, n, kind), B, cuda)


@pytest.mark.parametrize("B", BLOCKS)
def test_empty_tensor(orc, wclib, cuda, B):
    words = np.zeros(0, np.uint16)
    got = gpu_compress_escape(wclib, to_gpu_words(words, cuda), B)
    assert np.array_equal(got, orc.compress_escape(words, B))
    dec, status = gpu_decompress_escape(wclib, got, 0, B, cuda)
    assert status == 0 and dec.size == 0


@pytest.mark.parametrize("B", BLOCKS)
def test_all_bf16_patterns(orc, wclib, cuda, B):
    roundtrip_vs_oracle(orc, wclib, np.arange(65536, dtype=np.uint16), B, cuda)
    permuted = np.random.default_rng(3).permutation(65536).astype(np.uint16)
    roundtrip_vs_oracle(orc, wclib, permuted, B, cuda)


def workload_cases():
    from lossless_weight_compression_b200 import synth
    for cfg in (1, 2, 5):
        for B in synth.WORKLOADS[cfg].blocks:
            yield cfg, B


@pytest.mark.parametrize("cfg,B", list(workload_cases()))
def test_workloads_vs_oracle(orc, wclib, cuda, cfg, B):
    from lossless_weight_compression_b200 import synth
    for _, t in synth.WORKLOADS[cfg].make(cuda):
        roundtrip_vs_oracle(orc, wclib, words_np(t), B, cuda)


def test_layer_workload_vs_oracle(orc, wclib, cuda):
    """One Llama-3-8B-shaped layer (218M elements), byte-exact per matrix."""
    from lossless_weight_compression_b200 import synth
    for _, t in synth.config3(cuda):
        roundtrip_vs_oracle(orc, wclib, words_np(t), 1024, cuda)


def test_determinism(wclib, cuda):
    from lossless_weight_compression_b200 import synth
    (_, t), = synth.config5(cuda)
    first = gpu_compress_escape(wclib, t, 256)
    for _ in range(2):
        assert np.array_equal(first, gpu_compress_escape(wclib, t, 256))


def test_batch_decode_spans_launches(wclib, cuda):
    """600 escape-coded streams of mixed sizes and block sizes in one call
    (two launches)."""
    rng = np.random.default_rng(21)
    items, pairs = [], []
    for k in range(600):
        n = int(rng.integers(0, 5000)) if k % 50 else 100_003
        B = BLOCKS[k % len(BLOCKS)]
        words = to_gpu_words(random_words(rng, n, "mixed" if k % 3 else "gauss"), cuda)
        c = wclib.compress_escape(words, B)
        out = torch.full((n,), -1, dtype=torch.int16, device=cuda)
        items.append((c.buffer, c.size(), out, n, B))
        pairs.append((words, out))
    status = torch.zeros(1, dtype=torch.int32, device=cuda)
    wclib.decompress_escape_batch(wclib.make_batch(items), status)
    torch.cuda.synchronize()
    assert status.item() == 0
    assert all(torch.equal(a, b) for a, b in pairs)


def test_kinds_do_not_mix(orc, wclib, cuda):
    """A plain stream given to the escape-coded decoder, and the other way
    round, is reported as corrupt."""
    from gpu_util import gpu_decompress
    words = random_words(np.random.default_rng(22), 20_000, "gauss")
    plain, esc = orc.compress(words, 512), orc.compress_escape(words, 512)
    _, st = gpu_decompress_escape(wclib, plain, words.size, 512, cuda)
    assert st == wclib.WC_ERR_CORRUPT_STREAM
    _, st = gpu_decompress(wclib, esc, words.size, 512, cuda)
    assert st == wclib.WC_ERR_CORRUPT_STREAM


def test_corrupt_escape_streams_are_reported(orc, wclib, cuda):
    B, words, good, _ = golden_io.load_kind("esc_w2_two_escapes.txt")
    n = words.size

    def status_of(s):
        return gpu_decompress_escape(wclib, s, n, B, cuda)[1]

    assert status_of(good) == 0
    cases = []
    s = good.copy(); s[129] = 9; cases.append(s)            # w = 9
    s = good.copy(); s[128] = 253; cases.append(s)          # base > 255 - (2^2 - 1)
    s = good.copy(); s[512:516] = 0xFF; cases.append(s)     # 16 escapes: no room for them
    s = good.copy(); s[12] = 0; cases.append(s)             # plain flags
    s = good.copy(); s[256] = 1; cases.append(s)            # offset of block 0
    for c in cases:
        assert status_of(c) == wclib.WC_ERR_CORRUPT_STREAM
    # a truncated stream: the host rejects it before launching or the kernel reports it
    s = torch.from_numpy(good[:520].copy()).to(cuda)
    status = torch.zeros(1, dtype=torch.int32, device=cuda)
    out = torch.empty(n, dtype=torch.int16, device=cuda)
    rc = wclib.wc_decompress_escape(s.data_ptr(), 520, out.data_ptr(), n, B, status.data_ptr(),
                                    torch.cuda.current_stream().cuda_stream)
    torch.cuda.synchronize()
    assert rc == wclib.WC_ERR_CORRUPT_STREAM or status.item() == wclib.WC_ERR_CORRUPT_STREAM


def test_random_metadata_corruption_leaves_device_healthy(orc, wclib, cuda):
    """200 random corruptions of block headers, offsets and exception bytes: the
    status is ok or corrupt, and the device keeps working."""
    rng = np.random.default_rng(23)
    words = random_words(rng, 3 * 8192 + 77, "outliers")
    B = 256
    good = orc.compress_escape(words, B)
    nb = -(-words.size // B)
    off_offs = int(good[40:48].view(np.uint64)[0])
    off_exp = int(good[56:64].view(np.uint64)[0])
    for _ in range(200):
        s = good.copy()
        where = int(rng.integers(0, 3))
        if where == 0:
            s[128 + int(rng.integers(0, 2 * nb))] = rng.integers(0, 256)
        elif where == 1:
            s[off_offs + int(rng.integers(0, 4 * nb))] = rng.integers(0, 256)
        else:
            s[off_exp + int(rng.integers(0, good.size - off_exp))] = rng.integers(0, 256)
        _, st = gpu_decompress_escape(wclib, s, words.size, B, cuda)
        assert st in (0, wclib.WC_ERR_CORRUPT_STREAM)
    dec, st = gpu_decompress_escape(wclib, good, words.size, B, cuda)
    assert st == 0 and np.array_equal(dec, words)


def test_batch_compress_matches_oracle(orc, wclib, cuda):
    """One wc_compress_escape_batch call over tensors of mixed sizes and block sizes
    (an empty one included): every stream equals the oracle's."""
    rng = np.random.default_rng(24)
    shapes = [(0, 256), (1, 128), (8191, 512), (8193, 4096), (100_003, 128), (1 << 20, 1024),
              (3 * 8192 + 5, 2048), (65536, 256)]
    words = [random_words(rng, n, KINDS[k % len(KINDS)]) for k, (n, _) in enumerate(shapes)]
    batch = wclib.CompressBatch([to_gpu_words(w, cuda) for w in words],
                                block=[B for _, B in shapes], escape=True)
    batch.run()
    torch.cuda.synchronize()
    sizes = batch.sizes()
    for j, ((n, B), w) in enumerate(zip(shapes, words)):
        got = batch.buffers[j][: sizes[j]].cpu().numpy()
        assert np.array_equal(got, orc.compress_escape(w, B)), (n, B)


def test_batch_compress_spans_launches(orc, wclib, cuda):
    """More tensors than one launch takes (700 > 512): each launch has its own
    part of the workspace."""
    rng = np.random.default_rng(25)
    words = [random_words(rng, int(rng.integers(0, 20000)), "mixed") for _ in range(700)]
    batch = wclib.CompressBatch([to_gpu_words(w, cuda) for w in words], block=256, escape=True)
    batch.run()
    torch.cuda.synchronize()
    sizes = batch.sizes()
    for j in range(0, 700, 7):
        got = batch.buffers[j][: sizes[j]].cpu().numpy()
        assert np.array_equal(got, orc.compress_escape(words[j], 256))


def test_torch_helpers_round_trip_either_kind(wclib, cuda):
    w = torch.randn(1000, 777, device=cuda).mul_(0.02).to(torch.bfloat16)
    for c in (wclib.compress(w, 512), wclib.compress_escape(w, 512)):
        y = wclib.decompress_compressed(c)
        torch.cuda.synchronize()
        assert y.shape == w.shape and y.dtype == w.dtype
        assert torch.equal(y.view(torch.int16), w.view(torch.int16))
