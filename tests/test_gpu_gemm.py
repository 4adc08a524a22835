"""The fused decode + tensor-core matrix product (wc_gemm) against the oracle.

The oracle decodes its own stream and multiplies in float64; the GPU kernel is
fed the same stream (the GPU's own encoding, where a test compresses on the
GPU, is byte-identical by the parity tests, and the expected values still come
from the oracle's stream). Products of two BF16 values are exact in FP32; the
tensor cores accumulate in FP32 without a stated rounding mode, so the bound
held here is cols * 2^-22 * sum_c |W x| per output (four times the bound of a
round-to-nearest FP32 sum, enough for truncating accumulation with one guard
bit). Results must also be bitwise reproducible.
"""
import numpy as np
import pytest
import torch

from test_oracle_gemv import rand_bf16

pytestmark = pytest.mark.gpu

# (rows, cols, B): several 128-row units and 128-column slices, ragged row tails,
# blocks shorter and longer than a row (B = 4096 > cols: a block spans rows)
SHAPES = [(1, 128, 128), (7, 1024, 512), (130, 384, 128), (256, 4096, 1024),
          (300, 1280, 256), (129, 14336, 1024), (64, 2048, 4096), (200, 384, 256)]
TOKENS = [1, 16, 37, 64, 128]


def run_gpu(wc, stream_np, rows, cols, B, x_np, device, nbytes=None):
    s = torch.from_numpy(stream_np).to(device)
    x = torch.from_numpy(x_np.view(np.int16)).to(device)
    status = torch.zeros(1, dtype=torch.int32, device=device)
    y = wc.gemm(s, rows, cols, B, x, status=status, nbytes=nbytes)
    torch.cuda.synchronize()
    return y.cpu().numpy().astype(np.float64), int(status.item())


def check_bound(y, y_ref, absum, cols):
    tol = cols * 2.0 ** -22 * absum + 1e-30
    err = np.abs(y - y_ref)
    assert (err <= tol).all(), float((err / tol).max())


@pytest.mark.parametrize("rows,cols,B", SHAPES)
@pytest.mark.parametrize("tokens", TOKENS)
def test_gemm_matches_oracle(orc, wclib, cuda, rows, cols, B, tokens):
    rng = np.random.default_rng(rows * 131 + cols + tokens)
    W = rand_bf16(rng, (rows, cols), 0.02)
    x = rand_bf16(rng, (tokens, cols), 1.0)
    stream = orc.compress(W, B)
    y_ref, absum = orc.gemv(stream, rows, cols, B, x)
    y, status = run_gpu(wclib, stream, rows, cols, B, x, cuda)
    assert status == 0
    assert y.shape == (tokens, rows)
    check_bound(y, y_ref, absum, cols)
    y2, _ = run_gpu(wclib, stream, rows, cols, B, x, cuda)
    assert np.array_equal(y, y2)  # same bits every run


def test_gemm_raw_and_constant_blocks(orc, wclib, cuda):
    """Blocks of every width 0..8 in one matrix: constant rows (w = 0), exponents
    spread over [0, 130] (w = 8, stored raw), zeros and denormals."""
    rng = np.random.default_rng(50)
    rows, cols, B = 256, 1024, 256
    W = rand_bf16(rng, (rows, cols), 0.02)
    e = rng.integers(0, 131, size=(64, cols))
    s = rng.integers(0, 256, size=(64, cols))
    W[:64] = ((s & 0x80) << 8) | (e << 7) | (s & 0x7F)       # raw blocks, no overflow
    W[64:80] = 0x3F80                                          # 1.0 everywhere: w = 0
    W[80:96] = 0                                               # +0.0
    W[96:112] = rng.integers(0, 128, size=(16, cols))          # denormals: e = 0, w = 0
    for k in range(8):                                         # one row per width 1..8
        W[112 + k] = (rng.integers(100, 100 + min(1 << (k + 1), 129), size=cols) << 7) \
            | rng.integers(0, 128, size=cols)
    stream = orc.compress(W, B)
    x = rand_bf16(rng, (32, cols), 1.0)
    y_ref, absum = orc.gemv(stream, rows, cols, B, x)
    y, status = run_gpu(wclib, stream, rows, cols, B, x, cuda)
    assert status == 0
    finite = np.isfinite(y_ref) & (absum < 1e37)
    assert np.array_equal(np.isfinite(y), np.isfinite(y_ref))
    check_bound(y[finite], y_ref[finite], absum[finite], cols)


def test_gemm_with_special_values(orc, wclib, cuda):
    """NaN and Inf weights propagate as in exact arithmetic."""
    rng = np.random.default_rng(51)
    rows, cols, B = 130, 2048, 1024
    W = rand_bf16(rng, (rows, cols), 0.02)
    W[3, 5] = 0x7FC0     # NaN
    W[7, 100] = 0x7F80   # +Inf
    W[9, 7] = 0xFF80     # -Inf
    W[9, 8] = 0x7F80     # +Inf in the same row: Inf - Inf = NaN
    W[129, 2000] = 0xFF80
    x = rand_bf16(rng, (16, cols), 1.0)
    stream = orc.compress(W, B)
    y_ref, absum = orc.gemv(stream, rows, cols, B, x)
    y, status = run_gpu(wclib, stream, rows, cols, B, x, cuda)
    assert status == 0
    assert np.array_equal(np.isnan(y), np.isnan(y_ref))
    inf = np.isinf(y_ref)
    assert np.array_equal(y[inf], y_ref[inf])
    safe = np.isfinite(y_ref)
    check_bound(y[safe], y_ref[safe], absum[safe], cols)


def test_gemm_batch_over_several_launches(orc, wclib, cuda):
    """70 matrices of mixed shapes in one call (two launches of up to 64)."""
    rng = np.random.default_rng(52)
    items, refs = [], []
    tokens = 24
    for k in range(70):
        rows, cols, B = SHAPES[k % 6]
        rows = max(1, rows // 2 + k)
        W = rand_bf16(rng, (rows, cols), 0.02)
        x = rand_bf16(rng, (tokens, cols), 1.0)
        stream = orc.compress(W, B)
        refs.append(orc.gemv(stream, rows, cols, B, x) + (cols,))
        s = torch.from_numpy(stream).to(cuda)
        xt = torch.from_numpy(x.view(np.int16)).to(cuda)
        yt = torch.empty((tokens, rows), dtype=torch.float32, device=cuda)
        items.append((s, stream.size, xt, yt, rows, cols, B))
    status = torch.zeros(1, dtype=torch.int32, device=cuda)
    wclib.gemm_batch(wclib.make_gemv_batch(items), tokens, status)
    torch.cuda.synchronize()
    assert status.item() == 0
    for (s, sb, xt, yt, rows, cols, B), (y_ref, absum, cols_) in zip(items, refs):
        check_bound(yt.cpu().numpy().astype(np.float64), y_ref, absum, cols_)


def test_gemm_on_gpu_compressed_layer(orc, wclib, cuda):
    """A Llama-3-8B-shaped layer compressed on the GPU and multiplied with 64 tokens
    in one batched call; expected values from the oracle's own stream of the same
    seeded weights."""
    from lossless_weight_compression_b200 import synth
    rng = np.random.default_rng(53)
    tokens, B = 64, 1024
    items, refs = [], []
    for name, t in synth.layer_tensors(2, cuda):
        rows, cols = t.shape
        c = wclib.compress(t, B)
        x = rand_bf16(rng, (tokens, cols), 1.0)
        W = t.cpu().view(torch.int16).numpy().view(np.uint16)
        refs.append((name, cols) + orc.gemv(orc.compress(W, B), rows, cols, B, x))
        xt = torch.from_numpy(x.view(np.int16)).to(cuda)
        yt = torch.empty((tokens, rows), dtype=torch.float32, device=cuda)
        items.append((c.buffer, c.size(), xt, yt, rows, cols, B))
    status = torch.zeros(1, dtype=torch.int32, device=cuda)
    wclib.gemm_batch(wclib.make_gemv_batch(items), tokens, status)
    torch.cuda.synchronize()
    assert status.item() == 0
    for it, (name, cols, y_ref, absum) in zip(items, refs):
        y = it[3].cpu().numpy().astype(np.float64)
        err = np.abs(y - y_ref)
        assert (err <= cols * 2.0 ** -22 * absum).all(), name


def test_gemm_reports_corrupt_stream(orc, wclib, cuda):
    rng = np.random.default_rng(54)
    rows, cols, B = 200, 1024, 256
    stream = orc.compress(rand_bf16(rng, (rows, cols), 0.02), B)
    x = rand_bf16(rng, (16, cols), 1.0)
    bad = stream.copy()
    bad[128 + 2 * 5 + 1] = 9  # block 5: w = 9
    _, status = run_gpu(wclib, bad, rows, cols, B, x, cuda)
    assert status == 3
    bad = stream.copy()
    nb = rows * cols // B
    off_offs = 128 + (2 * nb + 127) // 128 * 128
    bad[off_offs + 4 * 7: off_offs + 4 * 8] = np.frombuffer(np.uint32(1 << 30).tobytes(), np.uint8)
    _, status = run_gpu(wclib, bad, rows, cols, B, x, cuda)  # offset far past the end
    assert status == 3
    bad = stream.copy()
    bad[0] ^= 1  # magic
    _, status = run_gpu(wclib, bad, rows, cols, B, x, cuda)
    assert status == 3
    # shorter than the exponent plane's offset: refused on the host
    s = torch.from_numpy(stream).to(cuda)
    xt = torch.from_numpy(x.view(np.int16)).to(cuda)
    with pytest.raises(RuntimeError):
        wclib.gemm(s, rows, cols, B, xt, nbytes=1000)
    # a stream cut inside its exponent plane: the payload bounds check catches it
    _, status = run_gpu(wclib, stream, rows, cols, B, x, cuda, nbytes=stream.size - 64)
    assert status == 3
    # the device is still usable
    y_ref, absum = orc.gemv(stream, rows, cols, B, x)
    y, status = run_gpu(wclib, stream, rows, cols, B, x, cuda)
    assert status == 0
    check_bound(y, y_ref, absum, cols)


def test_gemm_refuses_escape_coded_stream(orc, wclib, cuda):
    """The fused product decodes plain streams only: an escape-coded stream of the
    same matrix is reported as corrupt (its container header carries the escape
    flag), every read staying inside the stream, and the device stays usable."""
    rng = np.random.default_rng(55)
    rows, cols, B = 256, 1024, 512
    W = rand_bf16(rng, (rows, cols), 0.02)
    x = rand_bf16(rng, (16, cols), 1.0)
    esc = orc.compress_escape(W.reshape(-1), B)
    _, status = run_gpu(wclib, esc, rows, cols, B, x, cuda)
    assert status == 3
    stream = orc.compress(W, B)
    y_ref, absum = orc.gemv(stream, rows, cols, B, x)
    y, status = run_gpu(wclib, stream, rows, cols, B, x, cuda)
    assert status == 0
    check_bound(y, y_ref, absum, cols)


# ---------------------------------------------------------------------------
# escape-coded streams through wc_gemm_batch_flags
# ---------------------------------------------------------------------------
def esc_reference(orc, stream, rows, cols, B, x):
    """float64 product of the oracle's decode of an escape-coded stream."""
    from oracle import bf16_to_f64
    W = bf16_to_f64(orc.decompress_escape(stream, rows * cols, B)).reshape(rows, cols)
    xf = bf16_to_f64(np.asarray(x, dtype=np.uint16).reshape(-1, cols))
    with np.errstate(invalid="ignore", over="ignore"):
        return xf @ W.T, np.abs(xf) @ np.abs(W).T


def run_gpu_escape(wc, stream_np, rows, cols, B, x_np, device, nbytes=None):
    s = torch.from_numpy(stream_np).to(device)
    x = torch.from_numpy(x_np.view(np.int16)).to(device)
    y = torch.empty((x_np.shape[0], rows), dtype=torch.float32, device=device)
    status = torch.zeros(1, dtype=torch.int32, device=device)
    batch = wc.make_gemv_batch([(s, stream_np.size if nbytes is None else nbytes, x, y, rows, cols,
                                 B)])
    wc.gemm_batch(batch, x_np.shape[0], status, escape=True)
    torch.cuda.synchronize()
    return y.cpu().numpy().astype(np.float64), int(status.item())


@pytest.mark.parametrize("rows,cols,B", [(7, 1024, 512), (130, 384, 128), (256, 4096, 1024),
                                         (129, 14336, 1024), (64, 4096, 4096)])
@pytest.mark.parametrize("tokens", [1, 16, 64, 128])
def test_gemm_escape_coded_matches_oracle(orc, wclib, cuda, rows, cols, B, tokens):
    rng = np.random.default_rng(rows * 17 + cols + tokens)
    W = rand_bf16(rng, (rows, cols), 0.02)
    W[rng.random((rows, cols)) < 0.002] = 0x4580  # outliers: exceptions in most blocks
    x = rand_bf16(rng, (tokens, cols), 1.0)
    stream = orc.compress_escape(W.reshape(-1), B)
    y_ref, absum = esc_reference(orc, stream, rows, cols, B, x)
    y, status = run_gpu_escape(wclib, stream, rows, cols, B, x, cuda)
    assert status == 0
    check_bound(y, y_ref, absum, cols)
    y2, _ = run_gpu_escape(wclib, stream, rows, cols, B, x, cuda)
    assert np.array_equal(y, y2)


def test_gemm_escape_coded_arguments_and_kinds(orc, wclib, cuda):
    """Rows that are not whole blocks and unknown flags are refused on the host;
    a plain stream multiplied as escape-coded (and the reverse) is corrupt."""
    rng = np.random.default_rng(62)
    rows, cols, B = 64, 1024, 512
    W = rand_bf16(rng, (rows, cols), 0.02)
    x = rand_bf16(rng, (16, cols), 1.0)
    esc = orc.compress_escape(W.reshape(-1), B)
    s = torch.from_numpy(esc).to(cuda)
    xt = torch.from_numpy(x.view(np.int16)).to(cuda)
    y = torch.empty((16, rows), dtype=torch.float32, device=cuda)
    status = torch.zeros(1, dtype=torch.int32, device=cuda)
    arr, n = wclib.make_gemv_batch([(s, esc.size, xt, y, rows, cols, 2048)])  # 1024 % 2048 != 0
    assert wclib.wc_gemm_batch_flags(arr, n, 16, 2, status.data_ptr(), None) == wclib.WC_ERR_INVALID_ARG
    arr, n = wclib.make_gemv_batch([(s, esc.size, xt, y, rows, cols, B)])
    assert wclib.wc_gemm_batch_flags(arr, n, 16, 1, status.data_ptr(), None) == wclib.WC_ERR_INVALID_ARG
    _, st = run_gpu_escape(wclib, orc.compress(W, B), rows, cols, B, x, cuda)
    assert st == 3
    _, st = run_gpu(wclib, esc, rows, cols, B, x, cuda)
    assert st == 3
    y_ref, absum = esc_reference(orc, esc, rows, cols, B, x)
    yy, st = run_gpu_escape(wclib, esc, rows, cols, B, x, cuda)
    assert st == 0
    check_bound(yy, y_ref, absum, cols)


def test_gemm_escape_coded_reports_corruption(orc, wclib, cuda):
    """Corrupt escape-coded streams are reported and every read stays inside
    the stream; the device stays usable."""
    rng = np.random.default_rng(63)
    rows, cols, B = 128, 1024, 256
    W = rand_bf16(rng, (rows, cols), 0.02)
    W[rng.random((rows, cols)) < 0.01] = 0x4580
    x = rand_bf16(rng, (16, cols), 1.0)
    esc = orc.compress_escape(W.reshape(-1), B)
    nb = rows * cols // B
    hdr = esc[128:128 + 2 * nb].view(np.uint16)
    off_offs = 128 + (2 * nb + 127) // 128 * 128
    off_exp = off_offs + (4 * nb + 127) // 128 * 128 + rows * cols
    offs = esc[off_offs:off_offs + 4 * nb].view(np.uint32)
    psize = 16 * np.diff(offs.astype(np.int64))
    b = int(np.flatnonzero(((hdr[:-1] >> 8) == 3) & (psize > (B // 8) * 3))[0])  # w = 3, K >= 1
    cases = []
    bad = esc.copy()
    bad[128 + 2 * b] = 255                      # base above 255 - (2^w - 1)
    cases.append(bad)
    bad = esc.copy()
    bad[128 + 2 * b + 1] = 9                    # w = 9
    cases.append(bad)
    bad = esc.copy()
    start = off_exp + 16 * int(offs[b]) + (B // 8) * 3
    bad[start] = hdr[b] & 0xFF                  # an exception inside the window
    cases.append(bad)
    bad = esc.copy()
    bad[off_offs + 4 * 1: off_offs + 8] = np.frombuffer(np.uint32(1 << 28).tobytes(), np.uint8)
    cases.append(bad)                           # offset far past the end
    for k, bad in enumerate(cases):
        _, st = run_gpu_escape(wclib, bad, rows, cols, B, x, cuda)
        assert st == 3, k
    _, st = run_gpu_escape(wclib, esc, rows, cols, B, x, cuda, nbytes=esc.size - 32)
    assert st == 3
    y_ref, absum = esc_reference(orc, esc, rows, cols, B, x)
    y, st = run_gpu_escape(wclib, esc, rows, cols, B, x, cuda)
    assert st == 0
    check_bound(y, y_ref, absum, cols)
