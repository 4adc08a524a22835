"""GPU parity for the other dtypes: FP32 streams (wc_compress_fp32 /
wc_decompress_fp32) and FP16 words through the 16-bit path, against the CPU
oracle. The bar is the same as for BF16: the GPU stream equals the oracle's
byte for byte and the GPU decode gives back the input bits.
"""
import numpy as np
import pytest
import torch

from gpu_util import gpu_compress, gpu_decompress, to_gpu_words

pytestmark = pytest.mark.gpu


def fp32_words(rng, n, kind):
    if kind == "gauss":
        return (rng.standard_normal(n).astype(np.float32) * 0.02).view(np.uint32)
    if kind == "random":
        return rng.integers(0, 2 ** 32, n, dtype=np.uint64).astype(np.uint32)
    if kind == "mixed":
        w = fp32_words(rng, n, "gauss")
        if n:
            pos = rng.integers(0, n, max(1, n // 40))
            w[pos] = rng.choice(np.array([0, 0x80000000, 0x7F800000, 0xFF800000, 0x7FC00001,
                                          0xFFFFFFFF, 1, 0x807FFFFF], dtype=np.uint32), pos.size)
            a = int(rng.integers(0, n))
            w[a:a + 500] = rng.integers(0, 2 ** 32, len(w[a:a + 500]), dtype=np.uint64)
        return w
    raise ValueError(kind)


def gpu_compress_fp32(wc, words: np.ndarray, B: int, device):
    x = torch.from_numpy(words.view(np.int32).copy()).to(device)
    c = wc.compress_fp32(x, B)
    torch.cuda.synchronize()
    assert int(c.status.item()) == 0
    return c.stream().cpu().numpy()


def gpu_decompress_fp32(wc, stream: np.ndarray, n: int, B: int, device, nbytes=None):
    s = torch.from_numpy(np.ascontiguousarray(stream)).to(device)
    status = torch.zeros(1, dtype=torch.int32, device=device)
    out = torch.empty(n, dtype=torch.int32, device=device)
    wc.decompress_fp32(s, n, B, out=out, status=status,
                       nbytes=stream.size if nbytes is None else nbytes)
    torch.cuda.synchronize()
    return out.cpu().numpy().view(np.uint32), int(status.item())


@pytest.mark.parametrize("B", [128, 512, 1024, 4096])
@pytest.mark.parametrize("kind", ["gauss", "random", "mixed"])
def test_fp32_streams_match_oracle(orc, wclib, cuda, B, kind):
    rng = np.random.default_rng(B * 7 + len(kind))
    for n in (0, 1, 3, 7, 8, 9, 1000, 8191, 8192, 8193, 3 * 8192 + 5, 100000):
        x = fp32_words(rng, n, kind)
        ref = orc.compress_f32(x, B)
        got = gpu_compress_fp32(wclib, x, B, cuda)
        assert got.size == ref.size, (n, got.size, ref.size)
        diff = np.nonzero(got != ref)[0]
        assert diff.size == 0, (n, diff[:8])
        dec, status = gpu_decompress_fp32(wclib, ref, n, B, cuda)
        assert status == 0 and np.array_equal(dec, x), n


def test_fp32_layer_sized_tensor(orc, wclib, cuda):
    """A 4096 x 14336 FP32 matrix (235 MB, many tiles): stream equal to the oracle's,
    round trip on the device, ratio as the closed form predicts (> 1.1)."""
    g = torch.Generator(device=cuda)
    g.manual_seed(5)
    t = torch.randn((4096, 14336), generator=g, device=cuda) * 0.02
    x = t.view(-1).view(torch.int32).cpu().numpy().view(np.uint32)
    c = wclib.compress_fp32(t, 1024)
    torch.cuda.synchronize()
    assert int(c.status.item()) == 0
    ref = orc.compress_f32(x, 1024)
    got = c.stream().cpu().numpy()
    assert np.array_equal(got, ref)
    out = wclib.decompress_fp32(c.buffer, t.numel(), 1024, nbytes=c.size())
    torch.cuda.synchronize()
    assert torch.equal(out.view(-1).view(torch.int32), t.view(-1).view(torch.int32))
    assert 4 * t.numel() / c.size() > 1.1


def test_fp32_and_bf16_streams_are_not_interchangeable(orc, wclib, cuda):
    rng = np.random.default_rng(3)
    n, B = 20000, 512
    x = fp32_words(rng, n, "gauss")
    s32 = orc.compress_f32(x, B)
    _, status = gpu_decompress(wclib, s32, n, B, cuda)
    assert status == 3
    s16 = orc.compress((x >> 16).astype(np.uint16), B)
    try:  # too short for an FP32 layout: refused on the host, or by the kernel's checks
        _, status = gpu_decompress_fp32(wclib, s16, n, B, cuda)
    except wclib.WcodecError as e:
        status = e.status
    assert status == 3
    for pos in (12, 80, 81, 120):
        bad = s32.copy()
        bad[pos] ^= 1
        _, status = gpu_decompress_fp32(wclib, bad, n, B, cuda)
        assert status == 3, pos
    # the device is still usable
    dec, status = gpu_decompress_fp32(wclib, s32, n, B, cuda)
    assert status == 0 and np.array_equal(dec, x)


@pytest.mark.parametrize("B", [256, 1024])
def test_fp16_words_through_the_16_bit_path(orc, wclib, cuda, B):
    """FP16 tensors use wc_compress / wc_decompress unchanged: byte-exact against the
    oracle, round trip, and a ratio above 1 for Gaussian weights."""
    g = torch.Generator(device=cuda)
    g.manual_seed(B)
    t = (torch.randn(3 * 8192 + 77, generator=g, device=cuda) * 0.02).to(torch.float16)
    words = t.view(torch.int16).cpu().numpy().view(np.uint16)
    got, _ = gpu_compress(wclib, t.view(torch.int16), B)
    ref = orc.compress(words, B)
    assert np.array_equal(got, ref)
    dec, status = gpu_decompress(wclib, ref, words.size, B, cuda)
    assert status == 0 and np.array_equal(dec, words)
    assert 2 * words.size / ref.size > 1.03
