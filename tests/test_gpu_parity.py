"""GPU parity: libwcodec's CUDA encoder and decoder against the CPU oracle.

The bar is bit-exactness: the GPU's stream must equal the oracle's byte for
byte (header and zero padding included) and the GPU's decode must give back
the input words bit for bit, on every workload, at edge sizes and for every
block size. All calls go through the C-ABI library.
"""
import numpy as np
import pytest
import torch

import golden_io
from gpu_util import gpu_compress, gpu_decompress, to_gpu_words, words_np

pytestmark = pytest.mark.gpu

BLOCKS = (128, 256, 512, 1024, 2048, 4096)


def random_words(rng, n, kind):
    if kind == "gauss":
        f = (rng.standard_normal(n) * 0.02).astype(np.float32)
        return (f.view(np.uint32) >> 16).astype(np.uint16)
    if kind == "uniform":
        return rng.integers(0, 65536, n).astype(np.uint16)
    if kind == "zeros":
        return np.zeros(n, np.uint16)
    if kind == "narrow":
        return ((rng.integers(120, 124, n) << 7) | rng.integers(0, 65536, n) & 0x807F).astype(np.uint16)
    if kind == "mixed":  # gaussian with random specials and short random slabs
        w = random_words(rng, n, "gauss")
        if n:
            pos = rng.integers(0, n, max(1, n // 50))
            w[pos] = rng.choice([0x0000, 0x8000, 0x7F80, 0xFF80, 0x7FC0, 0xFFFF, 0x0001, 0x807F], pos.size)
            a = int(rng.integers(0, n))
            w[a:a + 300] = rng.integers(0, 65536, len(w[a:a + 300]))
        return w
    raise ValueError(kind)


def roundtrip_vs_oracle(orc, wc, words, B, device):
    ref = orc.compress(words, B)
    got, _ = gpu_compress(wc, to_gpu_words(words, device), B)
    assert got.size == ref.size, (got.size, ref.size)
    diff = np.nonzero(got != ref)[0]
    assert diff.size == 0, "first differing bytes at %s" % diff[:8]
    dec, status = gpu_decompress(wc, ref, words.size, B, device)
    assert status == 0
    assert np.array_equal(dec, words)


@pytest.mark.parametrize("name", golden_io.names())
def test_hand_derived_streams(wclib, cuda, name):
    B, words, expected = golden_io.load(name)
    got, _ = gpu_compress(wclib, to_gpu_words(words, cuda), B)
    assert np.array_equal(got, expected)
    dec, status = gpu_decompress(wclib, expected, words.size, B, cuda)
    assert status == 0 and np.array_equal(dec, words)


SIZES = [1, 7, 8, 9, 15, 16, 17, 127, 128, 129, 1000, 4095, 4096, 4097, 8191, 8192, 8193,
         3 * 8192 + 5, 100_003, 1 << 20]


KINDS = ["gauss", "uniform", "zeros", "narrow", "mixed"]


@pytest.mark.parametrize("B", BLOCKS)
@pytest.mark.parametrize("kind", KINDS)
def test_edge_sizes_vs_oracle(orc, wclib, cuda, B, kind):
    rng = np.random.default_rng(10 * B + KINDS.index(kind))
    for n in SIZES + [B - 1, B + 1, 5 * B + 3]:
        roundtrip_vs_oracle(orc, wclib, random_words(rng, n, kind), B, cuda)


@pytest.mark.parametrize("B", BLOCKS)
def test_empty_tensor(orc, wclib, cuda, B):
    words = np.zeros(0, np.uint16)
    got, _ = gpu_compress(wclib, to_gpu_words(words, cuda), B)
    assert np.array_equal(got, orc.compress(words, B))
    dec, status = gpu_decompress(wclib, got, 0, B, cuda)
    assert status == 0 and dec.size == 0


@pytest.mark.parametrize("B", BLOCKS)
def test_all_bf16_patterns(orc, wclib, cuda, B):
    natural = np.arange(65536, dtype=np.uint16)
    roundtrip_vs_oracle(orc, wclib, natural, B, cuda)
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


def test_config5_raw_slab_takes_raw_path(wclib, cuda):
    """Every block entirely inside the uniform-random slab is stored raw."""
    from lossless_weight_compression_b200 import synth
    (_, t), = synth.config5(cuda)
    start, length = synth.CFG5_RANDOM_SLAB
    for B in BLOCKS:
        stream, _ = gpu_compress(wclib, t, B)
        nb = -(-t.numel() // B)
        w = stream[128:128 + 2 * nb].view(np.uint16) >> 8
        first, last = -(-start // B), (start + length) // B  # blocks fully inside
        assert (w[first:last] == 8).all()


def test_layer_workload_vs_oracle(orc, wclib, cuda):
    """One Llama-3-8B-shaped layer (218M elements), byte-exact per matrix."""
    from lossless_weight_compression_b200 import synth
    for _, t in synth.config3(cuda):
        roundtrip_vs_oracle(orc, wclib, words_np(t), 1024, cuda)


def test_determinism(wclib, cuda):
    from lossless_weight_compression_b200 import synth
    (_, t), = synth.config5(cuda)
    first, _ = gpu_compress(wclib, t, 256)
    for _ in range(3):
        again, _ = gpu_compress(wclib, t, 256)
        assert np.array_equal(first, again)


def test_batch_decode_matches_inputs(wclib, cuda):
    rng = np.random.default_rng(9)
    tensors, items = [], []
    for k, (n, B) in enumerate([(0, 128), (1, 256), (8193, 512), (100_000, 4096), (777, 128),
                                (1 << 20, 1024), (65536 * 3 + 1, 2048)]):
        words = to_gpu_words(random_words(rng, n, "mixed"), cuda)
        c = wclib.compress(words, B)
        out = torch.full((n,), -1, dtype=torch.int16, device=cuda)
        tensors.append((words, out))
        items.append((c.buffer, c.size(), out, n, B))
    status = torch.zeros(1, dtype=torch.int32, device=cuda)
    wclib.decompress_batch(wclib.make_batch(items), status)
    torch.cuda.synchronize()
    assert status.item() == 0
    for words, out in tensors:
        assert torch.equal(words, out)


def test_many_item_batch_spans_launches(wclib, cuda):
    """More items than one launch holds: the library splits the batch."""
    rng = np.random.default_rng(10)
    n_items = 600
    items, pairs = [], []
    for k in range(n_items):
        n = int(rng.integers(0, 3000))
        words = to_gpu_words(random_words(rng, n, "gauss"), cuda)
        c = wclib.compress(words, 128)
        out = torch.empty(n, dtype=torch.int16, device=cuda)
        items.append((c.buffer, c.size(), out, n, 128))
        pairs.append((words, out))
    status = torch.zeros(1, dtype=torch.int32, device=cuda)
    wclib.decompress_batch(wclib.make_batch(items), status)
    torch.cuda.synchronize()
    assert status.item() == 0
    assert all(torch.equal(a, b) for a, b in pairs)


def test_batch_compress_matches_oracle(orc, wclib, cuda):
    """One wc_compress_batch call over tensors of mixed sizes and block sizes
    (including an empty one): every stream equals the oracle's."""
    rng = np.random.default_rng(12)
    shapes = [(0, 256), (1, 128), (8191, 512), (8193, 4096), (100_003, 128), (1 << 20, 1024),
              (3 * 8192 + 5, 2048), (65536, 256)]
    words = [random_words(rng, n, "mixed") for n, _ in shapes]
    tensors = [to_gpu_words(w, cuda) for w in words]
    batch = wclib.CompressBatch(tensors, block=[B for _, B in shapes])
    batch.run()
    torch.cuda.synchronize()
    assert batch.status.item() == 0
    for j, ((n, B), w) in enumerate(zip(shapes, words)):
        got = batch.buffers[j][: batch.sizes()[j]].cpu().numpy()
        assert np.array_equal(got, orc.compress(w, B)), (n, B)


def test_batch_compress_spans_launches(orc, wclib, cuda):
    """More tensors than one launch takes: each launch has its own workspace part."""
    rng = np.random.default_rng(13)
    words = [random_words(rng, int(rng.integers(0, 20000)), "gauss") for _ in range(700)]
    batch = wclib.CompressBatch([to_gpu_words(w, cuda) for w in words], block=128)
    batch.run()
    torch.cuda.synchronize()
    assert batch.status.item() == 0
    sizes = batch.sizes()
    for j in range(0, 700, 7):
        got = batch.buffers[j][: sizes[j]].cpu().numpy()
        assert np.array_equal(got, orc.compress(words[j], 128))


def test_stack_shaped_batch_round_trip(wclib, cuda):
    """A batch shaped like one decoder layer plus a ragged tensor, compressed in
    one call and decoded in one call, gives back every tensor bit for bit."""
    from lossless_weight_compression_b200 import synth
    tensors = [t.view(-1).view(torch.int16) for _, t in synth.layer_tensors(3, cuda)]
    tensors.append(to_gpu_words(random_words(np.random.default_rng(14), 123_457, "mixed"), cuda))
    batch = wclib.CompressBatch(tensors, block=1024)
    batch.run()
    torch.cuda.synchronize()
    assert batch.status.item() == 0
    sizes = batch.sizes()
    outs = [torch.empty_like(t) for t in tensors]
    status = torch.zeros(1, dtype=torch.int32, device=cuda)
    wclib.decompress_batch(wclib.make_batch(
        [(batch.buffers[j], sizes[j], outs[j], t.numel(), 1024) for j, t in enumerate(tensors)]),
        status)
    torch.cuda.synchronize()
    assert status.item() == 0
    assert all(torch.equal(a, b) for a, b in zip(tensors, outs))
