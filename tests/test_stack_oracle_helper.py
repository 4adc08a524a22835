"""The thread-pool comparison the full-size parity tests use, on the CPU: it
must report a stream that differs in one byte or in length, and nothing else."""
import numpy as np
import torch

from stack_oracle import compare_all


def test_compare_all_finds_planted_differences(orc):
    rng = np.random.default_rng(9)
    items, planted = [], set()
    for k in range(12):
        n = int(rng.integers(1, 40000))
        w = (rng.standard_normal(n) * 0.02).astype(np.float32)
        words = (w.view(np.uint32) >> 16).astype(np.uint16)
        s = orc.compress(words, 256).copy()
        if k % 4 == 1:
            s[int(rng.integers(128, s.size))] ^= 0x10
            planted.add("t%d" % k)
        if k % 4 == 3:
            s = np.concatenate([s, np.zeros(16, np.uint8)])
            planted.add("t%d" % k)
        items.append(("t%d" % k, torch.from_numpy(words.view(np.int16)), torch.from_numpy(s)))
    # a small budget forces the main thread to wait for jobs to finish
    bad, count = compare_all(iter(items), lambda x: orc.compress(x, 256),
                             max_bytes_in_flight=200_000)
    assert count == 12
    assert set(bad) == planted
