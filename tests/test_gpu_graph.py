"""The batched entry points inside a CUDA graph.

The library neither allocates nor synchronizes on its launch paths, and the
batch descriptors travel as launch parameters, so a captured batch can be
replayed: the replays must give the same bytes as direct calls. Each entry
point is called once directly first (its one-time, per-device set-up runs
outside the capture). All calls go through the C-ABI.
"""
import numpy as np
import pytest
import torch

from gpu_util import to_gpu_words

pytestmark = pytest.mark.gpu


def words(rng, n):
    f = (rng.standard_normal(n) * 0.02).astype(np.float32)
    return (f.view(np.uint32) >> 16).astype(np.uint16)


@pytest.mark.parametrize("escape", [False, True])
def test_captured_compress_and_decode_batches_replay(wclib, cuda, escape):
    rng = np.random.default_rng(41)
    tensors = [to_gpu_words(words(rng, n), cuda) for n in (5000, 1 << 20, 123_457, 8192)]
    enc = wclib.CompressBatch(tensors, block=1024, escape=escape)
    enc.run()  # direct call: set-up and the reference streams
    torch.cuda.synchronize()
    sizes = enc.sizes()
    ref = [enc.buffers[k][:sizes[k]].clone() for k in range(len(tensors))]
    outs = [torch.full_like(t, -1) for t in tensors]
    status = torch.zeros(1, dtype=torch.int32, device=cuda)
    batch = wclib.make_batch([(enc.buffers[k], sizes[k], outs[k], t.numel(), 1024)
                              for k, t in enumerate(tensors)])
    dec = wclib.decompress_escape_batch if escape else wclib.decompress_batch
    dec(batch, status)
    torch.cuda.synchronize()

    side = torch.cuda.Stream(cuda)
    side.wait_stream(torch.cuda.current_stream())
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.stream(side):
        with torch.cuda.graph(graph, stream=side):
            enc.run()
            dec(batch, status)
    torch.cuda.current_stream().wait_stream(side)
    for _ in range(2):
        for o in outs:
            o.fill_(-1)
        for b in enc.buffers:
            b.fill_(0)
        graph.replay()
        torch.cuda.synchronize()
        assert status.item() == 0 and enc.status.item() == 0
        assert enc.sizes() == sizes
        for k, t in enumerate(tensors):
            assert torch.equal(enc.buffers[k][:sizes[k]], ref[k])
            assert torch.equal(outs[k], t)
    del graph
