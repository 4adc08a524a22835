"""The fused decode + matrix-vector kernel (wc_gemv) against the oracle.

The oracle decodes its own stream and multiplies in float64; the GPU kernel is
fed the same stream. FP32 products of two BF16 values are exact, so the only
error is the FP32 summation, bounded by (cols - 1) * 2^-24 * sum_c |W x|; the
test holds every output to that bound. Results must also be bitwise
reproducible (the summation order is fixed).
"""
import numpy as np
import pytest
import torch

from test_oracle_gemv import rand_bf16

pytestmark = pytest.mark.gpu

SHAPES = [(1, 128, 128), (7, 1024, 512), (64, 4096, 1024), (33, 14336, 1024),
          (5, 9216, 1024), (3, 16384, 4096), (129, 256, 128), (1000, 2048, 2048)]


def run_gpu(wc, stream_np, rows, cols, B, x_np, device):
    s = torch.from_numpy(stream_np).to(device)
    x = torch.from_numpy(x_np.view(np.int16)).to(device)
    status = torch.zeros(1, dtype=torch.int32, device=device)
    y = wc.gemv(s, rows, cols, B, x, status=status)
    torch.cuda.synchronize()
    return y.cpu().numpy().astype(np.float64), int(status.item())


def check_bound(y, y_ref, absum, cols):
    tol = (cols - 1) * 2.0 ** -24 * absum + 1e-30
    err = np.abs(y - y_ref)
    assert (err <= tol).all(), float((err / tol).max())


@pytest.mark.parametrize("rows,cols,B", SHAPES)
@pytest.mark.parametrize("n_vec", [1, 2, 4])
def test_gemv_matches_oracle(orc, wclib, cuda, rows, cols, B, n_vec):
    rng = np.random.default_rng(rows * 131 + cols + n_vec)
    W = rand_bf16(rng, (rows, cols), 0.02)
    x = rand_bf16(rng, (n_vec, cols), 1.0)
    stream = orc.compress(W, B)
    y_ref, absum = orc.gemv(stream, rows, cols, B, x)
    y, status = run_gpu(wclib, stream, rows, cols, B, x, cuda)
    assert status == 0
    check_bound(y, y_ref, absum, cols)
    y2, _ = run_gpu(wclib, stream, rows, cols, B, x, cuda)
    assert np.array_equal(y, y2)  # same bits every run


def test_gemv_with_special_values(orc, wclib, cuda):
    """NaN and Inf weights propagate as in exact arithmetic; finite rows that cannot
    overflow in FP32 stay within the bound."""
    rng = np.random.default_rng(40)
    rows, cols, B = 64, 2048, 256
    W = rand_bf16(rng, (rows, cols), 0.02)
    W[3, 5] = 0x7FC0     # NaN
    W[7, 100] = 0x7F80   # +Inf
    W[9, 7] = 0xFF80     # -Inf
    W[9, 8] = 0x7F80     # +Inf in the same row: Inf - Inf = NaN
    W[11, :300] = rng.integers(0, 65536, 300)  # raw, possibly huge values
    x = rand_bf16(rng, (1, cols), 1.0)
    stream = orc.compress(W, B)
    y_ref, absum = orc.gemv(stream, rows, cols, B, x)
    y, status = run_gpu(wclib, stream, rows, cols, B, x, cuda)
    assert status == 0
    assert np.array_equal(np.isnan(y), np.isnan(y_ref))
    inf = np.isinf(y_ref)
    assert np.array_equal(y[inf], y_ref[inf])
    safe = np.isfinite(y_ref) & (absum < 1e37)
    check_bound(y[safe], y_ref[safe], absum[safe], cols)


def test_gemv_batch_matches_single_calls(orc, wclib, cuda):
    rng = np.random.default_rng(41)
    items, refs = [], []
    for rows, cols, B in SHAPES[:6]:
        W = rand_bf16(rng, (rows, cols), 0.02)
        x = rand_bf16(rng, (2, cols), 1.0)
        stream = orc.compress(W, B)
        refs.append(orc.gemv(stream, rows, cols, B, x) + (cols,))
        s = torch.from_numpy(stream).to(cuda)
        xt = torch.from_numpy(x.view(np.int16)).to(cuda)
        yt = torch.empty((2, rows), dtype=torch.float32, device=cuda)
        items.append((s, stream.size, xt, yt, rows, cols, B))
    status = torch.zeros(1, dtype=torch.int32, device=cuda)
    wclib.gemv_batch(wclib.make_gemv_batch(items), 2, status)
    torch.cuda.synchronize()
    assert status.item() == 0
    for (s, sb, xt, yt, rows, cols, B), (y_ref, absum, cols_) in zip(items, refs):
        check_bound(yt.cpu().numpy().astype(np.float64), y_ref, absum, cols_)


def test_gemv_on_gpu_compressed_layer(wclib, cuda):
    """A Llama-3-8B-shaped layer compressed on the GPU: the fused product equals the
    product with the decoded weights (torch, FP64) within the FP32 bound."""
    from lossless_weight_compression_b200 import synth
    g = torch.Generator(device=cuda)
    g.manual_seed(42)
    for name, t in synth.layer_tensors(1, cuda):
        rows, cols = t.shape
        c = wclib.compress(t, 1024)
        x = torch.randn((1, cols), generator=g, device=cuda).to(torch.bfloat16)
        status = torch.zeros(1, dtype=torch.int32, device=cuda)
        y = wclib.gemv(c.buffer, rows, cols, 1024, x, nbytes=c.size(), status=status)
        ref = (x.double() @ t.double().T)
        absum = (x.double().abs() @ t.double().abs().T)
        torch.cuda.synchronize()
        assert status.item() == 0
        assert ((y.double() - ref).abs() <= (cols - 1) * 2.0 ** -24 * absum).all(), name


def test_gemv_reports_corrupt_stream(orc, wclib, cuda):
    rng = np.random.default_rng(43)
    rows, cols, B = 16, 1024, 256
    stream = orc.compress(rand_bf16(rng, (rows, cols), 0.02), B)
    bad = stream.copy()
    bad[128 + 2 * 5 + 1] = 9  # block 5: w = 9
    _, status = run_gpu(wclib, bad, rows, cols, B, rand_bf16(rng, (1, cols), 1.0), cuda)
    assert status == 3


def test_gemv_refuses_escape_coded_stream(orc, wclib, cuda):
    """Plain streams only: an escape-coded stream of the same matrix is reported as
    corrupt, and the device stays usable."""
    rng = np.random.default_rng(44)
    rows, cols, B = 64, 2048, 1024
    W = rand_bf16(rng, (rows, cols), 0.02)
    x = rand_bf16(rng, (1, cols), 1.0)
    _, status = run_gpu(wclib, orc.compress_escape(W.reshape(-1), B), rows, cols, B, x, cuda)
    assert status == 3
    stream = orc.compress(W, B)
    y_ref, absum = orc.gemv(stream, rows, cols, B, x)
    y, status = run_gpu(wclib, stream, rows, cols, B, x, cuda)
    assert status == 0
    check_bound(y, y_ref, absum, cols)
