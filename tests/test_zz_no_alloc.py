"""wc_compress_noalloc, the allocation-free encoder entry point, against wc_compress
and the oracle.

Callers that cannot allocate device memory -- an engine that has reserved the
GPU's memory for its own pools, or a path that must not stall on the device
synchronisation cudaMalloc/cudaFree may imply -- use wc_compress_noalloc,
which keeps the encoder's look-back state in a fixed array inside the library
instead of a caller workspace. Its stream must be byte-for-byte the stream
wc_compress writes for the same input and the oracle's stream of it (the codec
is integer work, so the tolerance is zero), on two calls in a row: the second
call reuses the array the first one left behind. Everything goes through the
C-ABI.

This file is named to be collected last.
"""
import numpy as np
import pytest
import torch

pytestmark = pytest.mark.gpu


def _inputs(device):
    rng = np.random.default_rng(2024)
    a = (rng.standard_normal(3 * 8192 + 77) * 0.02).astype(np.float32)
    a = (a.view(np.uint32) >> 16).astype(np.uint16)
    b = rng.integers(0, 65536, (1 << 20) + 13).astype(np.uint16)  # mostly raw blocks
    b[: 1 << 19] = a[0]                                           # and a long w = 0 run
    return [(torch.from_numpy(a.view(np.int16)).to(device), 512),
            (torch.from_numpy(b.view(np.int16)).to(device), 128)]


def _with_workspace(wc, x, block):
    c = wc.compress(x, block)
    torch.cuda.synchronize()
    assert c.status.item() == 0
    return c.stream().cpu().numpy()


def _noalloc(wc, x, block):
    n = x.numel()
    cap = wc.wc_bound(n, block)
    out = torch.empty((cap + 15) // 16 * 16, dtype=torch.uint8, device=x.device)
    nbytes = torch.zeros(1, dtype=torch.int64, device=x.device)
    status = torch.zeros(1, dtype=torch.int32, device=x.device)
    rc = wc.wc_compress_noalloc(x.data_ptr(), n, block, out.data_ptr(), out.numel(),
                                nbytes.data_ptr(), status.data_ptr(),
                                torch.cuda.current_stream().cuda_stream)
    assert rc == wc.WC_OK, wc.wc_status_string(rc)
    torch.cuda.synchronize()
    assert status.item() == 0
    return out[: int(nbytes.item())].cpu().numpy()


def test_noalloc_matches_workspace_entry_on_two_calls_in_a_row(orc, wclib, cuda):
    for x, block in _inputs(cuda):
        expected = _with_workspace(wclib, x, block)
        got = _noalloc(wclib, x, block)
        assert got.size == expected.size
        assert np.array_equal(got, expected)
        ref = orc.compress(x.cpu().numpy().view(np.uint16), block)
        assert np.array_equal(got, ref)


def test_noalloc_rejects_sizes_beyond_its_array(wclib, cuda):
    # refused before anything is looked up or enqueued, so the pointers are never used
    too_many = (1 << 30) + 1
    rc = wclib.wc_compress_noalloc(16, too_many, 1024, 16, 1 << 40, 16, None, None)
    assert rc == wclib.WC_ERR_BUFFER_TOO_SMALL
