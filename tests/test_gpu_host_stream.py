"""Decompression fused with the host-to-device transfer: streams in page-locked
host memory, decoded by wc_decompress_host[_batch] straight into device memory.

The compressed bytes cross the host link once, read by the decoder itself
("ENEC: A Lossless AI Model Compression Method Enabling Fast Inference on
Ascend NPUs", Abstract: compression cuts the transfer in weight-transfer-bound
inference). The bar is the decoder's: the output equals the input bit for bit,
for plain and escape-coded streams written by the CPU oracle, at ragged sizes
and every block size, in batches spanning several launches; corrupt streams end
in WC_ERR_CORRUPT_STREAM; pointers that are not page-locked host memory are
refused before anything is launched. All calls go through the C-ABI.
"""
import numpy as np
import pytest
import torch

pytestmark = pytest.mark.gpu

BLOCKS = (128, 256, 512, 1024, 2048, 4096)


def words_of(rng, n, kind):
    f = (rng.standard_normal(n) * 0.02).astype(np.float32)
    w = (f.view(np.uint32) >> 16).astype(np.uint16)
    if kind == "mixed" and n:
        pos = rng.integers(0, n, max(1, n // 50))
        w[pos] = rng.choice([0x0000, 0x8000, 0x7F80, 0xFF80, 0x7FC0, 0xFFFF, 0x0001], pos.size)
        a = int(rng.integers(0, n))
        w[a:a + 300] = rng.integers(0, 65536, len(w[a:a + 300]))
    return w


def pinned(a: np.ndarray) -> torch.Tensor:
    t = torch.empty(a.size, dtype=torch.uint8, pin_memory=True)
    t.copy_(torch.from_numpy(np.ascontiguousarray(a)))
    return t


def decode_host(wc, items, escape, device):
    """items: list of (host stream uint8 numpy, n, block); returns outputs, status."""
    hosts = [pinned(s) for s, _, _ in items]
    outs = [torch.full((n,), -1, dtype=torch.int16, device=device) for _, n, _ in items]
    status = torch.zeros(1, dtype=torch.int32, device=device)
    batch = wc.make_batch([(h, h.numel(), o, n, b) for h, o, (_, n, b) in zip(hosts, outs, items)])
    wc.decompress_host_batch(batch, status, escape=escape)
    torch.cuda.synchronize()
    return [o.cpu().numpy().view(np.uint16) for o in outs], int(status.item())


@pytest.mark.parametrize("escape", [False, True])
@pytest.mark.parametrize("B", BLOCKS)
def test_host_streams_decode_bit_exact(orc, wclib, cuda, escape, B):
    rng = np.random.default_rng(B + (7 if escape else 0))
    enc = orc.compress_escape if escape else orc.compress
    words = [words_of(rng, n, "mixed") for n in (1, 17, B - 1, B + 1, 8193, 100_003, 1 << 20)]
    outs, status = decode_host(wclib, [(enc(w, B), w.size, B) for w in words], escape, cuda)
    assert status == 0
    for w, o in zip(words, outs):
        assert np.array_equal(w, o)


def test_host_batch_spans_launches(orc, wclib, cuda):
    rng = np.random.default_rng(31)
    words = [words_of(rng, int(rng.integers(0, 4000)), "gauss") for _ in range(600)]
    outs, status = decode_host(wclib, [(orc.compress(w, 256), w.size, 256) for w in words],
                               False, cuda)
    assert status == 0
    assert all(np.array_equal(w, o) for w, o in zip(words, outs))


def test_host_stream_layer_round_trip(wclib, cuda):
    """The seven matrices of one Llama-3-8B-shaped layer, compressed on the GPU,
    moved to pinned host memory and decoded from there."""
    from lossless_weight_compression_b200 import synth
    ts = [t.view(-1).view(torch.int16) for _, t in synth.layer_tensors(0, cuda)]
    for escape in (False, True):
        comp = [wclib.compress_escape(t, 1024) if escape else wclib.compress(t, 1024) for t in ts]
        torch.cuda.synchronize()
        hosts = [c.stream().cpu().pin_memory() for c in comp]
        outs = [torch.empty_like(t) for t in ts]
        status = torch.zeros(1, dtype=torch.int32, device=cuda)
        batch = wclib.make_batch([(h, h.numel(), o, t.numel(), 1024)
                                  for h, o, t in zip(hosts, outs, ts)])
        wclib.decompress_host_batch(batch, status, escape=escape)
        torch.cuda.synchronize()
        assert status.item() == 0
        assert all(torch.equal(a, b) for a, b in zip(ts, outs))


def test_corrupt_host_stream_is_reported(orc, wclib, cuda):
    w = words_of(np.random.default_rng(32), 20_000, "gauss")
    s = orc.compress(w, 512)
    s[129] = 9  # block 0: w = 9
    _, status = decode_host(wclib, [(s, w.size, 512)], False, cuda)
    assert status == wclib.WC_ERR_CORRUPT_STREAM
    # an escape-coded stream read as a plain one, and the other way round
    _, status = decode_host(wclib, [(orc.compress_escape(w, 512), w.size, 512)], False, cuda)
    assert status == wclib.WC_ERR_CORRUPT_STREAM
    _, status = decode_host(wclib, [(orc.compress(w, 512), w.size, 512)], True, cuda)
    assert status == wclib.WC_ERR_CORRUPT_STREAM


def test_only_page_locked_host_memory_is_taken(orc, wclib, cuda):
    w = words_of(np.random.default_rng(33), 5000, "gauss")
    s = orc.compress(w, 256)
    out = torch.empty(w.size, dtype=torch.int16, device=cuda)
    status = torch.zeros(1, dtype=torch.int32, device=cuda)
    sh = torch.cuda.current_stream().cuda_stream
    dev = torch.from_numpy(s).to(cuda)  # device memory: use wc_decompress
    assert wclib.wc_decompress_host(dev.data_ptr(), s.size, out.data_ptr(), w.size, 256, 0,
                                    status.data_ptr(), sh) == wclib.WC_ERR_INVALID_ARG
    pageable = np.zeros(s.size + 16, np.uint8)  # ordinary host memory, 16-byte aligned view
    off = (-pageable.ctypes.data) % 16
    pageable[off:off + s.size] = s
    assert wclib.wc_decompress_host(pageable.ctypes.data + off, s.size, out.data_ptr(), w.size, 256,
                                    0, status.data_ptr(), sh) == wclib.WC_ERR_INVALID_ARG
    torch.cuda.synchronize()
    assert status.item() == 0  # nothing ran
