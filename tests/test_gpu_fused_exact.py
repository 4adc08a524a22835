"""The fused products' decoding, pinned exactly by one-hot activations.

With activation row t equal to the unit vector e_c (BF16 1.0 at column c, +0.0
elsewhere), Y[t][r] = sum_c' W[r][c'] * x[t][c'] has one product W[r][c] * 1.0
and every other term is a signed zero, so for finite weights the FP32 result is
W[r][c] exactly, whatever the order or rounding of the accumulation. Sending
every column of W through such rows turns the output into W transposed: it must
equal, value for value, the oracle's decode of the oracle's own stream, which
is also the stream the kernels read. A single wrongly decoded weight anywhere
fails, which the FP32 error bound of random activations cannot promise at wide
rows.

Shapes: the ragged ones of the bound tests (row tails, blocks shorter and
longer than a row, every 128-column slice) and a full Llama-3-8B-shaped layer
(cols 4096 and 14336, the widths of the benchmark). The tensor-core product is
also run on escape-coded streams (wc_gemm_batch_flags), whose expected weights
are the oracle's decode of its own escape-coded stream.
"""
import numpy as np
import pytest
import torch

from test_oracle_gemv import rand_bf16

pytestmark = pytest.mark.gpu

# (rows, cols, B); the GEMM takes cols in multiples of 128, the GEMV cols in
# multiples of B
GEMM_SHAPES = [(1, 128, 128), (7, 1024, 512), (130, 384, 128), (256, 4096, 1024),
               (300, 1280, 256), (129, 14336, 1024), (64, 2048, 4096), (200, 384, 256),
               (33, 9216, 2048)]
GEMV_SHAPES = [(1, 128, 128), (7, 1024, 512), (64, 4096, 1024), (33, 14336, 1024),
               (5, 9216, 1024), (3, 16384, 4096), (129, 256, 128), (1000, 2048, 2048)]
# escape-coded streams: rows of whole blocks
ESC_SHAPES = [(1, 128, 128), (7, 1024, 512), (130, 384, 128), (256, 4096, 1024),
              (300, 1280, 256), (129, 14336, 1024), (64, 4096, 4096), (200, 512, 256)]


def decoded_f32(orc, stream, rows, cols, B, escape=False):
    dec = orc.decompress_escape if escape else orc.decompress
    w = dec(stream, rows * cols, B).reshape(rows, cols)
    return (w.astype(np.uint32) << 16).view(np.float32)


def one_hot(cols, device):
    x = torch.zeros((cols, cols), dtype=torch.bfloat16, device=device)
    x.fill_diagonal_(1.0)
    return x


def run_one_hot(wc, kind, s_dev, size, rows, cols, B, device, per_call, columns=None,
                escape=False):
    """Y (len(columns) x rows) with row j the product of e_{columns[j]}."""
    cols_idx = np.arange(cols) if columns is None else np.asarray(columns)
    eye = one_hot(cols, device)
    X = eye[torch.from_numpy(cols_idx).to(device)].contiguous()
    Y = torch.full((cols_idx.size, rows), float("nan"), dtype=torch.float32, device=device)
    items = []
    for j in range(0, cols_idx.size, per_call):
        k = min(per_call, cols_idx.size - j)
        items.append((k, (s_dev, size, X[j:j + k], Y[j:j + k], rows, cols, B)))
    status = torch.zeros(1, dtype=torch.int32, device=device)
    full = [it for k, it in items if k == per_call]
    tail = [it for k, it in items if k != per_call]
    if kind == "gemm":
        def batch_fn(batch, n, st):
            wc.gemm_batch(batch, n, st, escape=escape)
    else:
        batch_fn = wc.gemv_batch
    if full:
        batch_fn(wc.make_gemv_batch(full), per_call, status)
    for s_, sz, x, y, r, c, b in tail:
        if kind == "gemm":
            batch_fn(wc.make_gemv_batch([(s_, sz, x, y, r, c, b)]), x.shape[0], status)
        else:  # the GEMV takes 1, 2 or 4 vectors: the tail one at a time
            for t in range(x.shape[0]):
                batch_fn(wc.make_gemv_batch([(s_, sz, x[t:t + 1], y[t:t + 1], r, c, b)]), 1,
                         status)
    torch.cuda.synchronize()
    assert status.item() == 0
    return Y.cpu().numpy(), cols_idx


def boundary_columns(cols, B, rng):
    """Both sides of every block edge inside a row, one column per 128-column
    slice, and the row's first and last columns."""
    c = {0, cols - 1}
    for e in range(B, cols, B):
        c.update((e - 1, e))
    for s in range(0, cols, 128):
        c.add(int(rng.integers(s, min(s + 128, cols))))
    return sorted(c)


@pytest.mark.parametrize("rows,cols,B", GEMM_SHAPES)
def test_gemm_one_hot_every_column(orc, wclib, cuda, rows, cols, B):
    rng = np.random.default_rng(rows * 7 + cols)
    W = rand_bf16(rng, (rows, cols), 0.02)
    stream = orc.compress(W, B)
    expect = decoded_f32(orc, stream, rows, cols, B)
    s = torch.from_numpy(stream).to(cuda)
    Y, _ = run_one_hot(wclib, "gemm", s, stream.size, rows, cols, B, cuda, 128)
    assert np.array_equal(Y.T, expect)


@pytest.mark.parametrize("rows,cols,B", GEMV_SHAPES)
@pytest.mark.parametrize("n_vec", [1, 2, 4])
def test_gemv_one_hot(orc, wclib, cuda, rows, cols, B, n_vec):
    rng = np.random.default_rng(rows * 11 + cols + n_vec)
    W = rand_bf16(rng, (rows, cols), 0.02)
    stream = orc.compress(W, B)
    expect = decoded_f32(orc, stream, rows, cols, B)
    s = torch.from_numpy(stream).to(cuda)
    columns = None if n_vec == 4 else boundary_columns(cols, B, rng)
    Y, idx = run_one_hot(wclib, "gemv", s, stream.size, rows, cols, B, cuda, n_vec, columns)
    assert np.array_equal(Y.T, expect[:, idx])


def test_gemm_one_hot_special_weights(orc, wclib, cuda):
    """Zeros, denormals, constant and raw blocks: the one-hot output is still the
    weight itself (finite weights only: 0 * Inf would be NaN)."""
    rng = np.random.default_rng(60)
    rows, cols, B = 256, 1024, 256
    W = rand_bf16(rng, (rows, cols), 0.02)
    e = rng.integers(0, 255, size=(64, cols))
    sm = rng.integers(0, 256, size=(64, cols))
    W[:64] = ((sm & 0x80) << 8) | (e << 7) | (sm & 0x7F)      # raw blocks, finite
    W[64:80] = 0x3F80
    W[80:96] = 0x8000                                          # -0.0
    W[96:112] = rng.integers(0, 128, size=(16, cols))          # denormals
    for k in range(8):
        W[112 + k] = (rng.integers(100, 100 + min(1 << (k + 1), 129), size=cols) << 7) \
            | rng.integers(0, 128, size=cols)
    stream = orc.compress(W, B)
    expect = decoded_f32(orc, stream, rows, cols, B)
    s = torch.from_numpy(stream).to(cuda)
    for kind, per in (("gemm", 128), ("gemv", 4)):
        Y, _ = run_one_hot(wclib, kind, s, stream.size, rows, cols, B, cuda, per)
        assert np.array_equal(Y.T, expect), kind


@pytest.mark.parametrize("rows,cols,B", ESC_SHAPES)
def test_gemm_one_hot_every_column_escape_coded(orc, wclib, cuda, rows, cols, B):
    rng = np.random.default_rng(rows * 13 + cols + B)
    W = rand_bf16(rng, (rows, cols), 0.02)
    stream = orc.compress_escape(W.reshape(-1), B)
    expect = decoded_f32(orc, stream, rows, cols, B, escape=True)
    s = torch.from_numpy(stream).to(cuda)
    Y, _ = run_one_hot(wclib, "gemm", s, stream.size, rows, cols, B, cuda, 128, escape=True)
    assert np.array_equal(Y.T, expect)


def test_gemm_one_hot_escape_coded_many_exceptions(orc, wclib, cuda):
    """Blocks of every kind in an escape-coded stream: long exception lists
    (exponents spread over the whole range in one element of ten, so that a
    block's list outgrows the bytes staged per row), constant rows (w = 0),
    raw rows (w = 8), zeros and denormals."""
    rng = np.random.default_rng(61)
    rows, cols, B = 256, 2048, 512
    W = rand_bf16(rng, (rows, cols), 0.02)
    pick = rng.random((64, cols)) < 0.1
    e = rng.integers(0, 255, size=(64, cols))
    sm = rng.integers(0, 256, size=(64, cols))
    W[:64] = np.where(pick, ((sm & 0x80) << 8) | (e << 7) | (sm & 0x7F), W[:64])
    e = rng.integers(0, 255, size=(16, cols))
    sm = rng.integers(0, 256, size=(16, cols))
    W[64:80] = ((sm & 0x80) << 8) | (e << 7) | (sm & 0x7F)    # raw blocks
    W[80:96] = 0x3F80
    W[96:112] = 0x8000
    W[112:128] = rng.integers(0, 128, size=(16, cols))
    stream = orc.compress_escape(W.reshape(-1), B)
    expect = decoded_f32(orc, stream, rows, cols, B, escape=True)
    s = torch.from_numpy(stream).to(cuda)
    Y, _ = run_one_hot(wclib, "gemm", s, stream.size, rows, cols, B, cuda, 128, escape=True)
    assert np.array_equal(Y.T, expect)


@pytest.fixture(scope="module")
def layer(orc, cuda):
    """A full Llama-3-8B-shaped layer, its oracle streams on the device and the
    oracle's decode of them."""
    from lossless_weight_compression_b200 import synth
    B = 1024
    out = []
    for name, t in synth.layer_tensors(4, "cpu"):
        rows, cols = t.shape
        W = t.view(torch.int16).numpy().view(np.uint16)
        stream = orc.compress(W, B)
        out.append((name, rows, cols, torch.from_numpy(stream).to(cuda), stream.size,
                    decoded_f32(orc, stream, rows, cols, B)))
    return B, out


@pytest.mark.parametrize("kind,per_call", [("gemm", 128), ("gemv", 4)])
def test_fused_one_hot_full_layer_every_weight(wclib, cuda, layer, kind, per_call):
    B, mats = layer
    for name, rows, cols, s, size, expect in mats:
        Y, _ = run_one_hot(wclib, kind, s, size, rows, cols, B, cuda, per_call)
        assert np.array_equal(Y.T, expect), name


def test_gemm_one_hot_full_layer_escape_coded(orc, wclib, cuda):
    """The same layer as escape-coded streams, every weight through the tensor cores."""
    from lossless_weight_compression_b200 import synth
    B = 1024
    for name, t in synth.layer_tensors(4, "cpu"):
        rows, cols = t.shape
        W = t.view(torch.int16).numpy().view(np.uint16).reshape(-1)
        stream = orc.compress_escape(W, B)
        expect = decoded_f32(orc, stream, rows, cols, B, escape=True)
        s = torch.from_numpy(stream).to(cuda)
        Y, _ = run_one_hot(wclib, "gemm", s, stream.size, rows, cols, B, cuda, 128, escape=True)
        assert np.array_equal(Y.T, expect), name
