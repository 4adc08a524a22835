"""tANS-coded streams on the GPU against the oracle, through the C-ABI: the
GPU encoder's stream byte for byte equal to the oracle's, and the GPU decoder
rebuilding the input bit for bit from the oracle's streams (integer work: the
tolerance is zero). The format is the reading of "MINE: Entropy-coded
Memory-efficient Inference for Large Language Models", Abstract, a
tANS-family GPU coder, that oracle/wc_oracle.c defines."""
import numpy as np
import pytest
import torch

import golden_io
from gpu_util import to_gpu_words

pytestmark = pytest.mark.gpu

CHUNKS = (1024, 2048, 4096, 8192)


def gauss_words(rng, n, std=0.02):
    f = (rng.standard_normal(n) * std).astype(np.float32)
    return (f.view(np.uint32) >> 16).astype(np.uint16)


def gpu_encode(wc, words_list, chunk, R, device):
    """One wc_compress_tans_batch call; returns the streams as host arrays."""
    ts = [to_gpu_words(w, device) if w.size else torch.empty(0, dtype=torch.int16, device=device)
          for w in words_list]
    enc = wc.CompressBatch(ts, block=chunk, tans_log=R)
    enc.run()
    torch.cuda.synchronize()
    sizes = enc.sizes()
    return [enc.buffers[k][:sizes[k]].cpu().numpy() for k in range(len(ts))]


def gpu_decode(wc, streams, ns, chunk, device):
    """One wc_decompress_tans_batch call; returns (host words, status)."""
    ss = [torch.from_numpy(np.ascontiguousarray(s)).to(device) for s in streams]
    outs = [torch.empty(max(n, 1), dtype=torch.int16, device=device) for n in ns]
    status = torch.zeros(1, dtype=torch.int32, device=device)
    wc.decompress_tans_batch(wc.make_batch(
        [(s, s.numel(), o, n, chunk) for s, o, n in zip(ss, outs, ns)]), status)
    torch.cuda.synchronize()
    return [o[:n].cpu().numpy().view(np.uint16) for o, n in zip(outs, ns)], int(status.item())


@pytest.mark.parametrize("name", ["tans_one_symbol.txt", "tans_two_symbols.txt"])
def test_hand_derived_streams(wclib, cuda, name):
    C, R, words, expected = golden_io.load_tans(name)
    got = gpu_encode(wclib, [words], C, R, cuda)[0]
    assert np.array_equal(got, expected)
    back, st = gpu_decode(wclib, [expected], [words.size], C, cuda)
    assert st == 0 and np.array_equal(back[0], words)


@pytest.mark.parametrize("C", CHUNKS)
@pytest.mark.parametrize("R", [8, 11, 12])
def test_edge_sizes_vs_oracle(orc, wclib, cuda, C, R):
    rng = np.random.default_rng(C + R)
    ns = [0, 1, 31, 32, 33, C - 1, C, C + 1, 3 * C + 77]
    words = [gauss_words(rng, n) for n in ns]
    words[-1][rng.integers(0, ns[-1], 50)] = rng.integers(0, 65536, 50)
    got = gpu_encode(wclib, words, C, R, cuda)
    for w, g in zip(words, got):
        ref = orc.compress_tans(w, C, R)
        assert g.size == ref.size and np.array_equal(g, ref), w.size
    back, st = gpu_decode(wclib, [orc.compress_tans(w, C, R) for w in words], ns, C, cuda)
    assert st == 0
    for w, b in zip(words, back):
        assert np.array_equal(w, b), w.size


@pytest.mark.parametrize("C", CHUNKS)
def test_every_pattern(orc, wclib, cuda, C):
    rng = np.random.default_rng(C)
    allw = np.arange(65536, dtype=np.uint16)
    for w in (allw, rng.permutation(allw)):
        ref = orc.compress_tans(w, C, 12)
        got = gpu_encode(wclib, [w], C, 12, cuda)[0]
        assert np.array_equal(got, ref)
        back, st = gpu_decode(wclib, [ref], [w.size], C, cuda)
        assert st == 0 and np.array_equal(back[0], w)


def test_many_tensors_in_one_batch(orc, wclib, cuda):
    """300 tensors (two launches of the decoder), many of one chunk each, so that
    the encoder's four-chunk groups straddle several tensors."""
    rng = np.random.default_rng(5)
    ns = [int(rng.integers(0, 3000)) if k % 3 else int(rng.integers(0, 40000)) for k in range(300)]
    words = [gauss_words(rng, n, 0.02 * (1 + k % 7)) for k, n in enumerate(ns)]
    got = gpu_encode(wclib, words, 1024, 11, cuda)
    refs = [orc.compress_tans(w, 1024, 11) for w in words]
    for k, (g, r) in enumerate(zip(got, refs)):
        assert np.array_equal(g, r), k
    back, st = gpu_decode(wclib, refs, ns, 1024, cuda)
    assert st == 0
    for w, b in zip(words, back):
        assert np.array_equal(w, b)


def test_layer_vs_oracle(orc, wclib, cuda):
    """A Llama-3-8B-shaped layer (218M elements) encoded on the GPU in one batch,
    every stream equal to the oracle's, decoded back on the GPU in one launch."""
    from lossless_weight_compression_b200 import synth
    from stack_oracle import compare_all
    C, R = 4096, 11
    names, ts = [], []
    for name, t in synth.layer_tensors(1, cuda):
        names.append(name)
        ts.append(t.view(-1).view(torch.int16))
    enc = wclib.CompressBatch(ts, block=C, tans_log=R)
    enc.run()
    torch.cuda.synchronize()
    sizes = enc.sizes()
    bad, count = compare_all(((names[k], ts[k], enc.buffers[k][:sizes[k]]) for k in range(len(ts))),
                             lambda w: orc.compress_tans(w, C, R))
    assert count == len(ts) and not bad, bad
    outs = [torch.empty_like(t) for t in ts]
    status = torch.zeros(1, dtype=torch.int32, device=cuda)
    wclib.decompress_tans_batch(wclib.make_batch(
        [(enc.buffers[k], sizes[k], outs[k], ts[k].numel(), C) for k in range(len(ts))]), status)
    torch.cuda.synchronize()
    assert status.item() == 0
    for name, a, b in zip(names, ts, outs):
        assert torch.equal(a, b), name


def test_stream_info(orc, wclib):
    w = np.arange(5000, dtype=np.uint16)
    s = orc.compress_tans(w, 2048, 10)
    n, block, total = wclib.stream_info(s[:128].tobytes())
    assert (n, block, total) == (5000, 2048, s.size)


def test_corrupt_streams_are_reported(orc, wclib, cuda):
    rng = np.random.default_rng(11)
    n, C = 3000, 1024
    w = gauss_words(rng, n)
    s = orc.compress_tans(w, C, 10)
    nb = -(-n // C)
    off_exp = 128 + 512 + (4 * nb + 127) // 128 * 128 + (n + 127) // 128 * 128
    cases = []
    b = s.copy(); b[12] = 5; cases.append(b)                    # flags
    b = s.copy(); b[88] = 13; cases.append(b)                   # table log out of range
    b = s.copy(); b[128 + 2 * 120] ^= 1; cases.append(b)        # counts no longer sum to L
    b = s.copy(); b[off_exp] ^= 0x04; cases.append(b)           # a lane's first state
    b = s.copy(); b[off_exp + 1] = 0xFF; cases.append(b)        # a state >= L
    b = s.copy(); b[off_exp + 70] ^= 0x10; cases.append(b)      # a word's bit
    b = s.copy(); b[128 + 512] = 1; cases.append(b)             # chunk offset
    b = s.copy(); b[128 + 512 + 4: 128 + 512 + 8] = 0xFF; cases.append(b)  # offset far past the end
    for k, b in enumerate(cases):
        _, st = gpu_decode(wclib, [b], [n], C, cuda)
        assert st == 3, k
    _, st = gpu_decode(wclib, [s[:-16]], [n], C, cuda)          # truncated
    assert st == 3
    for trial in range(100):                                    # random byte flips
        b = s.copy()
        b[int(rng.integers(0, b.size))] ^= int(rng.integers(1, 256))
        _, st = gpu_decode(wclib, [b], [n], C, cuda)
        assert st in (0, 3)
    back, st = gpu_decode(wclib, [s], [n], C, cuda)             # the device is still usable
    assert st == 0 and np.array_equal(back[0], w)


def test_corruption_verdict_matches_the_oracle(orc, wclib, cuda):
    """Byte flips anywhere, and many in the header, counts, offsets and chunk
    payloads: the GPU decoder reports a corrupt stream exactly when the oracle
    does (a flip in the mantissa plane corrupts nothing; one in an unused
    padding byte or a word does)."""
    rng = np.random.default_rng(12)
    n, C = 5000, 1024
    w = gauss_words(rng, n)
    s = orc.compress_tans(w, C, 11)
    nb = -(-n // C)
    off_man = 128 + 512 + (4 * nb + 127) // 128 * 128
    off_exp = off_man + (n + 127) // 128 * 128
    where = np.concatenate([rng.integers(0, s.size, 150), rng.integers(0, off_man, 100),
                            rng.integers(off_man + n, off_exp, 20),
                            rng.integers(off_exp, s.size, 250)])
    corrupt = 0
    for k, pos in enumerate(where):
        b = s.copy()
        b[int(pos)] ^= int(rng.integers(1, 256))
        rc, ref = orc.decompress_tans_status(b, n, C)
        got, st = gpu_decode(wclib, [b], [n], C, cuda)
        assert st == (0 if rc == 0 else 3), (k, int(pos), rc, st)
        if rc == 0:
            assert np.array_equal(got[0], ref), (k, int(pos))
        corrupt += rc != 0
    assert corrupt > 300


@pytest.mark.parametrize("C", CHUNKS)
def test_staged_and_unstaged_chunks_in_one_tensor(orc, wclib, cuda, C):
    """Chunks of Gaussian weights (payload about C/3 bytes, staged in shared
    memory) next to chunks of uniformly spread exponents (payload near C bytes,
    read from global memory), in one tensor and one launch."""
    rng = np.random.default_rng(C + 3)
    n = 9 * C + 123
    w = gauss_words(rng, n)
    for c in range(1, 10, 3):
        w[c * C:(c + 1) * C] = rng.integers(0, 65536, C)
    ref = orc.compress_tans(w, C, 12)
    got = gpu_encode(wclib, [w], C, 12, cuda)[0]
    assert np.array_equal(got, ref)
    back, st = gpu_decode(wclib, [ref], [n], C, cuda)
    assert st == 0 and np.array_equal(back[0], w)
