"""Helpers for the GPU tests: run libwcodec through its C-ABI on torch buffers."""
from __future__ import annotations

import numpy as np
import torch


def words_np(t: torch.Tensor) -> np.ndarray:
    """BF16 bit patterns of a tensor as a host uint16 array."""
    return t.detach().contiguous().view(-1).view(torch.int16).cpu().numpy().view(np.uint16)


def to_gpu_words(words: np.ndarray, device) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(words).view(np.int16).copy()).to(device)


def gpu_compress(wc, words: torch.Tensor, block: int, check_status: bool = True):
    """Compress int16/bf16 words on the GPU; returns (stream as host uint8, status)."""
    c = wc.compress(words, block)
    torch.cuda.synchronize()
    status = int(c.status.item())
    if check_status:
        assert status == 0, wc.wc_status_string(status)
    return c.stream().cpu().numpy(), status


def gpu_decompress(wc, stream: np.ndarray, n: int, block: int, device, stream_bytes=None):
    """Decode host stream bytes on the GPU; returns (host uint16 words, status)."""
    s = torch.from_numpy(np.ascontiguousarray(stream)).to(device)
    status = torch.zeros(1, dtype=torch.int32, device=device)
    out = torch.empty(n, dtype=torch.int16, device=device)
    wc.decompress(s, n, block, out=out, status=status,
                  nbytes=stream.size if stream_bytes is None else stream_bytes)
    torch.cuda.synchronize()
    return out.cpu().numpy().view(np.uint16), int(status.item())
