"""Parity at full size: the 8B-shaped stack (226 tensors, 8,029,995,008 elements,
16.06 GB BF16) compressed in one wc_compress_batch call and decoded in one
wc_decompress_batch call -- the launch configuration the benchmark times.

Checks:
(a) every one of the 226 streams byte for byte against the oracle's stream of
    the same tensor (the oracle runs tensor by tensor on a thread per host
    core, with bounded host memory);
(b) decode(encode(x)) == x for every tensor, bit for bit, on the device;
(c) every stream's size, E and block headers against the closed form, computed
    from per-block exponent min/max with plain PyTorch reductions;
(d) sampled blocks of every tensor byte for byte against the oracle's encoding
    of the block alone: a block's header and exponent payload do not depend on
    the rest of the tensor.
"""
import numpy as np
import pytest
import torch

pytestmark = pytest.mark.gpu

B = 1024


def A(x):
    return (x + 127) // 128 * 128


def closed_form(words: torch.Tensor):
    """(total, E, hdr) of a tensor's stream from per-block min/max (torch ops)."""
    n = words.numel()
    nb = -(-n // B)
    e = ((words.to(torch.int32) >> 7) & 0xFF)
    pad = nb * B - n
    if pad:
        e = torch.cat([e, e[-1:].expand(pad)])
    e = e.view(nb, B)
    lo, hi = e.amin(1), e.amax(1)
    d = (hi - lo).to(torch.int64)
    # bit length of d, exactly: the number of powers of two 1, 2, ..., 128 not above d
    powers = 2 ** torch.arange(8, device=words.device, dtype=torch.int64)
    w = (d.unsqueeze(1) >= powers).sum(1)
    base = torch.where(w == 8, torch.zeros_like(lo), lo).to(torch.int64)
    L = torch.full((nb,), B, dtype=torch.int64, device=words.device)
    L[-1] = n - (nb - 1) * B
    E = int(((L + 7) // 8 * w).sum().item())
    total = 128 + A(2 * nb) + A(4 * nb) + A(n) + E
    return total, E, (base | (w << 8)).to(torch.int32)


@pytest.fixture(scope="module")
def stack(wclib, cuda):
    from lossless_weight_compression_b200 import synth
    names, tensors = [], []
    for name, t in synth.stack_tensors(cuda):
        names.append(name)
        tensors.append(t.view(-1).view(torch.int16))
    enc = wclib.CompressBatch(tensors, block=B)
    enc.run()
    torch.cuda.synchronize()
    assert enc.status.item() == 0
    yield names, tensors, enc
    del enc, tensors
    torch.cuda.empty_cache()


def test_stack_every_stream_matches_oracle(orc, wclib, cuda, stack):
    from stack_oracle import compare_all
    names, tensors, enc = stack
    sizes = enc.sizes()
    items = ((names[k], tensors[k], enc.buffers[k][:sizes[k]]) for k in range(len(tensors)))
    bad, count = compare_all(items, lambda w: orc.compress(w, B))
    assert count == 226
    assert not bad, bad


def test_stack_round_trip_in_one_launch_each_way(wclib, cuda, stack):
    names, tensors, enc = stack
    sizes = enc.sizes()
    outs = [torch.empty_like(t) for t in tensors]
    status = torch.zeros(1, dtype=torch.int32, device=cuda)
    wclib.decompress_batch(wclib.make_batch(
        [(enc.buffers[k], sizes[k], outs[k], tensors[k].numel(), B) for k in range(len(tensors))]),
        status)
    torch.cuda.synchronize()
    assert status.item() == 0
    for name, a, b in zip(names, tensors, outs):
        assert torch.equal(a, b), name


def test_stack_sizes_and_headers_match_closed_form(wclib, cuda, stack):
    names, tensors, enc = stack
    sizes = enc.sizes()
    for k, (name, words) in enumerate(zip(names, tensors)):
        total, E, hdr = closed_form(words)
        assert sizes[k] == total, name
        head = enc.buffers[k][:128].cpu().numpy()
        assert int(head[64:72].view(np.uint64)[0]) == E, name
        nb = hdr.numel()
        got = enc.buffers[k][128:128 + 2 * nb].view(torch.int16).to(torch.int32) & 0xFFFF
        assert torch.equal(got, hdr), name


def test_stack_sampled_blocks_match_oracle(orc, wclib, cuda, stack):
    names, tensors, enc = stack
    rng = np.random.default_rng(2024)
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
            ref = orc.compress(block, B)  # one block: header at 128, payload after the planes
            ref_exp = 128 + A(2) + A(4) + A(B)
            size = ref.size - ref_exp
            assert int(buf[128 + 2 * b:130 + 2 * b].view(torch.int16).item()) & 0xFFFF == \
                int(ref[128:130].view(np.uint16)[0]), (name, b)
            start = off_exp + 16 * int(offs[b].item())
            got = buf[start:start + size].cpu().numpy()
            assert np.array_equal(got, ref[ref_exp:]), (name, b)
