"""Fault handling on the GPU, without faulting the GPU: corrupt streams are
rejected through the device status word (every read stays inside the given
buffers), and a look-back wait that can never be satisfied ends by itself
with WC_ERR_TIMEOUT, leaving the context usable."""
import numpy as np
import pytest
import torch

from gpu_util import gpu_compress, gpu_decompress, to_gpu_words

pytestmark = pytest.mark.gpu


def gaussian_words(n, seed=0):
    f = (np.random.default_rng(seed).standard_normal(n) * 0.02).astype(np.float32)
    return (f.view(np.uint32) >> 16).astype(np.uint16)


def layout(n, B):
    A = lambda x: (x + 127) // 128 * 128
    nb = -(-n // B)
    off_offs = 128 + A(2 * nb)
    off_man = off_offs + A(4 * nb)
    return nb, off_offs, off_man, off_man + A(n)


@pytest.fixture(scope="module")
def good(orc):
    n, B = 5 * 8192 + 77, 256
    words = gaussian_words(n)
    return words, B, orc.compress(words, B)


def status_of(wclib, cuda, stream, n, B, nbytes=None):
    dec, status = gpu_decompress(wclib, stream, n, B, cuda, stream_bytes=nbytes)
    return status, dec


def test_valid_stream_has_status_ok(wclib, cuda, good):
    words, B, s = good
    st, dec = status_of(wclib, cuda, s, words.size, B)
    assert st == 0 and np.array_equal(dec, words)


@pytest.mark.parametrize("what", ["magic", "version", "flags", "reserved", "w9", "raw_base",
                                  "offs", "offs_last", "E", "total"])
def test_corrupt_metadata_is_reported(wclib, cuda, good, what):
    words, B, s = good
    n = words.size
    nb, off_offs, off_man, off_exp = layout(n, B)
    c = s.copy()
    if what == "magic":
        c[1] ^= 0xFF
    elif what == "version":
        c[4] = 2
    elif what == "flags":
        c[12] = 1
    elif what == "reserved":
        c[100] = 7
    elif what == "w9":
        c[128 + 2 * 3 + 1] = 9            # block 3: w = 9
    elif what == "raw_base":
        c[128 + 2 * 3 + 1] = 8            # block 3: w = 8 with a nonzero base
        c[128 + 2 * 3] = 5
    elif what == "offs":
        c[off_offs + 4 * 40] += 1         # block 40 starts 16 bytes late
    elif what == "offs_last":
        c[off_offs + 4 * (nb - 1)] += 1
    elif what == "E":
        c[64] += 16
    elif what == "total":
        c[72] += 16
    st, _ = status_of(wclib, cuda, c, n, B)
    assert st == 3, what


def test_truncated_stream_is_reported(wclib, cuda, good):
    words, B, s = good
    st, _ = status_of(wclib, cuda, s, words.size, B, nbytes=s.size - 1)
    assert st == 3
    # shorter than the fixed sections: refused on the host before any launch
    from lossless_weight_compression_b200.wcodec import WcodecError
    with pytest.raises(WcodecError):
        status_of(wclib, cuda, s, words.size, B, nbytes=layout(words.size, B)[3] - 1)


def test_wrong_n_or_block_is_reported(wclib, cuda, good):
    words, B, s = good
    assert status_of(wclib, cuda, s, words.size - 1, B)[0] == 3
    assert status_of(wclib, cuda, s, words.size, 512)[0] == 3


def test_random_metadata_corruption_never_escapes(wclib, cuda, good):
    """Random byte flips in the header, block headers and offsets: the decode
    either reports the stream corrupt or decodes inside its buffers."""
    words, B, s = good
    rng = np.random.default_rng(11)
    _, _, off_man, _ = layout(words.size, B)
    seen = set()
    for _ in range(200):
        c = s.copy()
        for _ in range(int(rng.integers(1, 4))):
            c[int(rng.integers(0, off_man))] ^= int(rng.integers(1, 256))
        st, _ = status_of(wclib, cuda, c, words.size, B)
        assert st in (0, 3)
        seen.add(st)
    assert 3 in seen
    # the context is still healthy
    st, dec = status_of(wclib, cuda, s, words.size, B)
    assert st == 0 and np.array_equal(dec, words)


def test_lookback_wait_times_out(wclib, cuda):
    """No thread block takes tile 0, so tile 1 waits on a flag nothing sets;
    the bounded wait ends with WC_ERR_TIMEOUT and the device stays usable."""
    n, B = 4 * 8192 + 5, 512
    x = to_gpu_words(gaussian_words(n, 1), cuda)
    cap = wclib.wc_bound(n, B)
    out = torch.empty(cap, dtype=torch.uint8, device=cuda)
    nbytes = torch.full((1,), 12345, dtype=torch.int64, device=cuda)
    status = torch.zeros(1, dtype=torch.int32, device=cuda)
    ws = wclib.workspace_for(n, B, cuda)
    rc = wclib.wc_debug_compress_stalled(x.data_ptr(), n, B, out.data_ptr(), cap,
                                         nbytes.data_ptr(), ws.data_ptr(), ws.numel(),
                                         status.data_ptr(), 50_000_000,
                                         torch.cuda.current_stream().cuda_stream)
    assert rc == 0
    torch.cuda.synchronize()
    assert status.item() == wclib.WC_ERR_TIMEOUT
    assert nbytes.item() == 0
    # a normal call on the same device still works
    stream, st = gpu_compress(wclib, x, B)
    assert st == 0
    dec, st = gpu_decompress(wclib, stream, n, B, cuda)
    assert st == 0 and np.array_equal(dec, gaussian_words(n, 1))
