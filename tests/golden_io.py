"""Reader for the hand-derived stream fixtures in tests/golden/ (syntax in README.txt)."""
from __future__ import annotations

import os

import numpy as np

GOLDEN_DIR = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def _expand(tokens):
    out = []
    for tok in tokens:
        if "*" in tok:
            count, group = tok.split("*", 1)
            out += [int(h, 16) for h in group.split(",")] * int(count)
        else:
            out.append(int(tok, 16))
    return out


def load(name: str):
    """Returns (block, words uint16, expected stream uint8)."""
    block, words, expected, _ = load_kind(name)
    return block, words, expected


def load_kind(name: str):
    """Returns (block, words uint16, expected stream uint8, kind): kind is "plain",
    "escape" (an escape-coded stream, the fixture's "kind escape" line) or "tans"
    (a tANS-coded stream; its table log is read by load_tans)."""
    return _load(name)[:4]


def load_tans(name: str):
    """Returns (chunk size, table log R, words uint16, expected stream uint8)."""
    block, words, expected, kind, R = _load(name)
    assert kind == "tans"
    return block, R, words, expected


def _load(name: str):
    block = total = R = None
    kind = "plain"
    words, runs = [], []
    with open(os.path.join(GOLDEN_DIR, name)) as f:
        for line in f:
            line = line.split("#", 1)[0].strip()
            if not line:
                continue
            key, _, rest = line.partition(" ")
            if key == "kind":
                kind = rest.strip()
            elif key == "block":
                block = int(rest)
            elif key == "tablelog":
                R = int(rest)
            elif key == "words":
                words += _expand(rest.split())
            elif key == "total":
                total = int(rest)
            elif key == "at":
                off, _, data = rest.partition(":")
                runs.append((int(off), _expand(data.split())))
            else:
                raise ValueError("bad fixture line: %r" % line)
    expected = np.zeros(total, dtype=np.uint8)
    for off, data in runs:
        expected[off:off + len(data)] = data
    return block, np.array(words, dtype=np.uint16), expected, kind, R


def names(kind: str = "plain"):
    """Fixture files holding streams of the given kind."""
    files = sorted(f for f in os.listdir(GOLDEN_DIR) if f.endswith(".txt") and f != "README.txt")
    return [f for f in files if load_kind(f)[3] == kind]
