"""Every stream of a large workload against the oracle's, byte for byte.

The oracle is single-threaded C; its ctypes calls release the GIL, so a thread
pool runs one oracle encoding per host core, each on its own tensor. The main
thread copies a tensor and its GPU-written stream to the host only when the
bytes in flight leave room for them, so host memory stays bounded however
large the workload is.
"""
from __future__ import annotations

import os
import threading
from concurrent.futures import ThreadPoolExecutor

import numpy as np
import torch


def host_threads() -> int:
    try:
        return max(1, len(os.sched_getaffinity(0)))
    except AttributeError:
        return max(1, os.cpu_count() or 1)


class _Budget:
    def __init__(self, limit: int):
        self.limit, self.used = limit, 0
        self.cv = threading.Condition()

    def take(self, n: int):
        with self.cv:
            # a single item larger than the limit still runs, alone
            self.cv.wait_for(lambda: self.used == 0 or self.used + n <= self.limit)
            self.used += n

    def give(self, n: int):
        with self.cv:
            self.used -= n
            self.cv.notify_all()


def compare_all(items, encode, max_bytes_in_flight: int = 24 << 30):
    """items: (name, words (device int16 tensor), stream (device uint8 tensor,
    exactly the stream's bytes)); encode: the oracle encoder of host uint16 words.
    Returns the names whose oracle stream differs from the GPU's (empty when all
    are byte-identical) and the number of tensors compared."""
    budget = _Budget(max_bytes_in_flight)
    bad, count = [], 0

    def job(name, words, got, cost):
        try:
            ref = encode(words)
            return None if (ref.size == got.size and np.array_equal(ref, got)) else name
        finally:
            budget.give(cost)

    with ThreadPoolExecutor(max_workers=host_threads()) as pool:
        futures = []
        for name, words, stream in items:
            # host input + oracle stream + GPU stream, the oracle stream at its bound
            cost = 2 * words.numel() + 2 * stream.numel() + 2 * words.numel()
            budget.take(cost)
            w = words.detach().reshape(-1).view(torch.int16).cpu().numpy().view(np.uint16)
            g = stream.detach().cpu().numpy()
            futures.append(pool.submit(job, name, w, g, cost))
            count += 1
        for f in futures:
            r = f.result()
            if r is not None:
                bad.append(r)
    return bad, count
