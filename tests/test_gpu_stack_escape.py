"""Parity at full size for escape-coded streams: the 8B-shaped stack (226
tensors, 8,029,995,008 elements, 16.06 GB BF16) compressed by one
wc_compress_escape_batch call and decoded by one wc_decompress_escape_batch
call -- the launch configuration `bench.py --workload escape` times.

Checks:
(a) every one of the 226 streams byte for byte against the oracle's
    escape-coded stream of the same tensor (the oracle runs tensor by tensor on
    a thread per host core, with bounded host memory);
(b) decode(encode(x)) == x for every tensor, bit for bit, on the device;
(c) every block's width and base, every offset, E and every stream's size
    against the choice rule recomputed here with plain PyTorch reductions (a
    256-bin exponent histogram per block, every window of every width, ties to
    the smaller width and then the larger base);
(d) sampled blocks of every tensor byte for byte against the oracle's encoding
    of the block alone: a block's header and payload (codes, exception list,
    padding) do not depend on the rest of the tensor.
"""
import numpy as np
import pytest
import torch

pytestmark = pytest.mark.gpu

B = 1024


def A(x):
    return (x + 127) // 128 * 128


def rule(words: torch.Tensor):
    """(w, base, padded sizes) of every block of a tensor, by the choice rule."""
    n = words.numel()
    nb = -(-n // B)
    e = ((words.to(torch.int64) >> 7) & 0xFF)
    blk = torch.arange(n, device=words.device) // B
    hist = torch.zeros(nb * 256, dtype=torch.int32, device=words.device)
    hist.index_add_(0, blk * 256 + e, torch.ones_like(e, dtype=torch.int32))
    hist = hist.view(nb, 256)
    L = torch.full((nb,), B, dtype=torch.int64, device=words.device)
    L[-1] = n - (nb - 1) * B
    octets = (L + 7) // 8
    below = torch.zeros((nb, 257), dtype=torch.int64, device=words.device)
    below[:, 1:] = torch.cumsum(hist, 1)
    # candidates in order of preference for equal cost: w = 0, 1, ..., 7, raw
    INF = torch.iinfo(torch.int64).max // 4
    one_value = (hist == L[:, None]).any(1)
    best_cost = torch.where(one_value, torch.zeros_like(L), torch.full_like(L, INF))
    best_w = torch.zeros_like(L)
    best_base = torch.argmax(hist, 1).to(torch.int64)  # the single exponent, where there is one
    best_k = torch.zeros_like(L)
    for w in range(1, 8):
        m = 2 ** w - 1
        inside = below[:, m:256] - below[:, 0:256 - m]       # bases 0 .. 255 - m
        top = inside.amax(1)
        # the largest base among the windows of most elements
        hit = (torch.flip(inside, [1]) == top[:, None]).to(torch.uint8)
        idx = 255 - m - torch.argmax(hit, dim=1).to(torch.int64)  # argmax: the first maximum
        cost = octets * w + (L - top)
        better = cost < best_cost
        best_cost = torch.where(better, cost, best_cost)
        best_w = torch.where(better, torch.full_like(L, w), best_w)
        best_base = torch.where(better, idx, best_base)
        best_k = torch.where(better, L - top, best_k)
    raw = 8 * octets < best_cost
    best_w = torch.where(raw, torch.full_like(L, 8), best_w)
    best_base = torch.where(raw, torch.zeros_like(L), best_base)
    best_k = torch.where(raw, torch.zeros_like(L), best_k)
    sizes = (octets * best_w + best_k + 15) // 16 * 16
    return best_w, best_base, sizes


@pytest.fixture(scope="module")
def stack(wclib, cuda):
    from lossless_weight_compression_b200 import synth
    names, tensors = [], []
    for name, t in synth.stack_tensors(cuda):
        names.append(name)
        tensors.append(t.view(-1).view(torch.int16))
    enc = wclib.CompressBatch(tensors, block=B, escape=True)
    enc.run()
    torch.cuda.synchronize()
    assert enc.status.item() == 0
    yield names, tensors, enc
    del enc, tensors
    torch.cuda.empty_cache()


def test_escape_stack_every_stream_matches_oracle(orc, wclib, cuda, stack):
    from stack_oracle import compare_all
    names, tensors, enc = stack
    sizes = enc.sizes()
    items = ((names[k], tensors[k], enc.buffers[k][:sizes[k]]) for k in range(len(tensors)))
    bad, count = compare_all(items, lambda w: orc.compress_escape(w, B))
    assert count == 226
    assert not bad, bad


def test_escape_stack_round_trip_in_one_batch_each_way(wclib, cuda, stack):
    names, tensors, enc = stack
    sizes = enc.sizes()
    outs = [torch.empty_like(t) for t in tensors]
    status = torch.zeros(1, dtype=torch.int32, device=cuda)
    wclib.decompress_escape_batch(wclib.make_batch(
        [(enc.buffers[k], sizes[k], outs[k], tensors[k].numel(), B) for k in range(len(tensors))]),
        status)
    torch.cuda.synchronize()
    assert status.item() == 0
    for name, a, b in zip(names, tensors, outs):
        assert torch.equal(a, b), name


def test_escape_stack_headers_offsets_and_sizes_match_the_rule(wclib, cuda, stack):
    names, tensors, enc = stack
    sizes = enc.sizes()
    for k, (name, words) in enumerate(zip(names, tensors)):
        n = words.numel()
        nb = -(-n // B)
        w, base, psize = rule(words)
        buf = enc.buffers[k]
        hdr = buf[128:128 + 2 * nb].view(torch.int16).to(torch.int64) & 0xFFFF
        assert torch.equal(hdr & 0xFF, base), name
        assert torch.equal(hdr >> 8, w), name
        off_offs = 128 + A(2 * nb)
        offs = buf[off_offs:off_offs + 4 * nb].view(torch.int32).to(torch.int64)
        expect = torch.cumsum(psize, 0) - psize
        assert torch.equal(offs * 16, expect), name
        E = int(psize.sum().item())
        head = buf[:128].cpu().numpy()
        assert int(head[64:72].view(np.uint64)[0]) == E, name
        assert sizes[k] == off_offs + A(4 * nb) + A(n) + E, name


def test_escape_stack_sampled_blocks_match_oracle(orc, wclib, cuda, stack):
    names, tensors, enc = stack
    rng = np.random.default_rng(2025)
    for k, (name, words) in enumerate(zip(names, tensors)):
        n = words.numel()
        nb = -(-n // B)
        buf = enc.buffers[k]
        off_offs = 128 + A(2 * nb)
        off_exp = off_offs + A(4 * nb) + A(n)
        offs = buf[off_offs:off_offs + 4 * nb].view(torch.int32)
        for b in rng.choice(nb, size=4, replace=False):
            b = int(b)
            block = words[b * B:(b + 1) * B].cpu().numpy().view(np.uint16)
            ref = orc.compress_escape(block, B)  # one block: header at 128, payload after the planes
            ref_exp = 128 + A(2) + A(4) + A(B)
            size = ref.size - ref_exp
            assert int(buf[128 + 2 * b:130 + 2 * b].view(torch.int16).item()) & 0xFFFF == \
                int(ref[128:130].view(np.uint16)[0]), (name, b)
            start = off_exp + 16 * int(offs[b].item())
            got = buf[start:start + size].cpu().numpy()
            assert np.array_equal(got, ref[ref_exp:]), (name, b)
