"""Seeded synthetic BF16 weight tensors for the five workloads.

This module only draws random numbers; it holds none of the codec's arithmetic.
The tests and the benchmark use it to feed the same bytes to the CUDA library
and to the CPU oracle.

The shapes follow an 8B-parameter Llama-3-style decoder (hidden 4096,
grouped-query k/v of 1024 rows, MLP 14336, vocabulary 128256), because the
workloads are LLM weight tensors: a layer's seven linear weights, and a 32-layer
stack plus embedding and LM head. Values are Gaussian N(0, sigma) drawn in fp32
and rounded to BF16 (round-to-nearest-even by ``Tensor.to``), the usual shape
of trained LLM weights; the codec's parity never depends on the values.

Every generator takes a ``device``: CUDA generators for the large workloads,
the CPU generator for small ones. The same seed on two devices gives different
(but each deterministic) values; parity tests always hand the *same* tensor to
both sides.
"""
from __future__ import annotations

import math
from dataclasses import dataclass
from typing import Callable, Iterator

import torch

# (name, rows, cols) of one decoder layer's linear weights.
LLAMA3_8B_LAYER = (
    ("q_proj", 4096, 4096),
    ("k_proj", 1024, 4096),
    ("v_proj", 1024, 4096),
    ("o_proj", 4096, 4096),
    ("gate_proj", 14336, 4096),
    ("up_proj", 14336, 4096),
    ("down_proj", 4096, 14336),
)
LLAMA3_8B_LAYERS = 32
LLAMA3_8B_VOCAB = 128256
HIDDEN = 4096

LAYER_ELEMS = sum(r * c for _, r, c in LLAMA3_8B_LAYER)  # 218,103,808
STACK_ELEMS = LLAMA3_8B_LAYERS * LAYER_ELEMS + 2 * LLAMA3_8B_VOCAB * HIDDEN  # 8,029,995,008


def _gen(seed: int, device) -> torch.Generator:
    g = torch.Generator(device=torch.device(device))
    g.manual_seed(seed)
    return g


def gaussian(shape, std: float, seed: int, device="cpu", dtype=torch.bfloat16) -> torch.Tensor:
    """N(0, std) drawn in fp32 from ``seed`` and rounded to ``dtype`` (BF16, FP16 or
    FP32: the same draws for every dtype)."""
    g = _gen(seed, device)
    x = torch.randn(shape, generator=g, device=device, dtype=torch.float32)
    x.mul_(std)
    return x if dtype == torch.float32 else x.to(dtype)


def gaussian_bf16(shape, std: float, seed: int, device="cpu") -> torch.Tensor:
    """N(0, std) drawn in fp32 from ``seed`` and rounded to BF16."""
    return gaussian(shape, std, seed, device, torch.bfloat16)


def config1(device="cpu"):
    """1024x1024, N(0, 0.02), CPU generator seed 0 (moved to ``device``)."""
    return [("w1024", gaussian_bf16((1024, 1024), 0.02, 0, "cpu").to(device))]


def config2(device="cpu"):
    """4096x4096 with per-row std log-uniform in [0.005, 0.05] (seed 1); 0.1% of
    entries, drawn without replacement (seed 2), set to +/-20 sigma of their row
    with a random sign; 8 rows (seed 3) set to +0.0."""
    rows = cols = 4096
    g1 = _gen(1, device)
    u = torch.rand(rows, generator=g1, device=device, dtype=torch.float32)
    row_std = torch.exp(math.log(0.005) + u * (math.log(0.05) - math.log(0.005)))
    x = torch.randn((rows, cols), generator=g1, device=device, dtype=torch.float32)
    x.mul_(row_std[:, None])
    n = rows * cols
    n_out = round(0.001 * n)  # 16,777
    g2 = _gen(2, device)
    pos = torch.randperm(n, generator=g2, device=device)[:n_out]
    sign = torch.randint(0, 2, (n_out,), generator=g2, device=device).to(torch.float32) * 2 - 1
    flat = x.view(-1)
    flat[pos] = sign * 20.0 * row_std[pos // cols]
    g3 = _gen(3, device)
    zero_rows = torch.randperm(rows, generator=g3, device=device)[:8]
    x[zero_rows] = 0.0
    return [("w4096_outliers", x.to(torch.bfloat16))]


def layer_tensors(layer: int, device="cpu", seed_base: int = 10,
                  dtype=torch.bfloat16) -> Iterator[tuple[str, torch.Tensor]]:
    """The seven linear weights of one decoder layer. Matrix k of layer l uses
    seed ``seed_base + 16*l + k`` for its std jitter U[0.7, 1.3] and its values."""
    for k, (name, r, c) in enumerate(LLAMA3_8B_LAYER):
        seed = seed_base + 16 * layer + k
        jitter = 0.7 + 0.6 * torch.rand((), generator=_gen(seed, "cpu")).item()
        yield f"layers.{layer}.{name}", gaussian((r, c), 0.02 * jitter, seed, device, dtype)


def config3(device="cpu"):
    """One decoder layer (~218M elements), sigma = 0.02 * U[0.7, 1.3] per matrix."""
    return list(layer_tensors(0, device))


def stack_names() -> list[str]:
    names = ["embed_tokens"]
    for l in range(LLAMA3_8B_LAYERS):
        names += [f"layers.{l}.{name}" for name, _, _ in LLAMA3_8B_LAYER]
    return names + ["lm_head"]


def stack_tensors(device="cuda", seed_base: int = 10) -> Iterator[tuple[str, torch.Tensor]]:
    """The 226 tensors of the 8B-shaped stack, generated one at a time: the
    embedding (seed ``seed_base + 1000``), 32 layers, the LM head
    (``seed_base + 1001``), all N(0, 0.02) apart from the per-matrix jitter of
    the layers. ``seed_base`` lets each rank of a multi-GPU run draw its own."""
    yield "embed_tokens", gaussian_bf16((LLAMA3_8B_VOCAB, HIDDEN), 0.02, seed_base + 1000, device)
    for l in range(LLAMA3_8B_LAYERS):
        yield from layer_tensors(l, device, seed_base)
    yield "lm_head", gaussian_bf16((LLAMA3_8B_VOCAB, HIDDEN), 0.02, seed_base + 1001, device)


def config4(device="cuda"):
    return list(stack_tensors(device))


# Special BF16 bit patterns scattered through config 5.
SPECIAL_PATTERNS = (
    0x0000, 0x8000,  # +0, -0
    0x7F80, 0xFF80,  # +Inf, -Inf
    0x7FC0, 0xFFC0,  # quiet NaN, both signs
    0x7F81, 0x7FBF,  # signalling NaN payloads
    0xFFFF, 0x7FFF,  # all-ones payloads
    0x0001, 0x807F,  # smallest / largest denormal payloads
)

# Slabs of config 5: (first element, length). Starts are deliberately not
# multiples of 128 so that every slab edge falls inside a block at every B.
CFG5_SHAPE = (4096, 14336)
CFG5_RANDOM_SLAB = (3 * 2**20 + 77, 4096 * 14336 // 8)
CFG5_DENORMAL_SLAB = (40_000_003, 1_000_000)
CFG5_SPECIALS = 4096


def config5(device="cpu"):
    """4096x14336 N(0, 0.02) (seed 5) overwritten by: a slab of uniform-random
    16-bit patterns (~1/8 of the tensor, seed 6) that can only take the raw
    path; a slab of denormals (exponent 0, random nonzero mantissa, both
    signs, seed 7); and 4096 scattered specials (+/-0, +/-Inf, NaN payloads)
    at random positions (seed 8)."""
    x = gaussian_bf16(CFG5_SHAPE, 0.02, 5, device)
    flat = x.view(-1).view(torch.int16)
    start, length = CFG5_RANDOM_SLAB
    flat[start:start + length] = torch.randint(
        -32768, 32768, (length,), generator=_gen(6, device), device=device, dtype=torch.int32
    ).to(torch.int16)
    start, length = CFG5_DENORMAL_SLAB
    g7 = _gen(7, device)
    mant = torch.randint(1, 128, (length,), generator=g7, device=device, dtype=torch.int32)
    sign = torch.randint(0, 2, (length,), generator=g7, device=device, dtype=torch.int32)
    # the 16-bit pattern sign<<15 | mantissa, written as a signed int16
    flat[start:start + length] = ((mant | (sign << 15)) - (sign << 16)).to(torch.int16)
    g8 = _gen(8, device)
    pos = torch.randperm(flat.numel(), generator=g8, device=device)[:CFG5_SPECIALS]
    which = torch.randint(0, len(SPECIAL_PATTERNS), (CFG5_SPECIALS,), generator=g8, device=device)
    table = torch.tensor([p - 65536 if p >= 32768 else p for p in SPECIAL_PATTERNS],
                         dtype=torch.int16, device=device)
    flat[pos] = table[which]
    return [("w4096x14336_mixed", x)]


@dataclass(frozen=True)
class Workload:
    name: str
    blocks: tuple[int, ...]
    make: Callable[..., list]
    description: str


WORKLOADS = {
    1: Workload("gaussian_1024x1024", (512,), config1,
                "single BF16 tensor 1024x1024, N(0, 0.02), seed 0, B=512"),
    2: Workload("rowscaled_outliers_4096x4096", (256, 1024), config2,
                "BF16 4096x4096, per-row std log-uniform [0.005, 0.05], 0.1% outliers at "
                "+/-20 sigma, 8 zero rows, B in {256, 1024}"),
    3: Workload("llama3_8b_layer", (1024,), config3,
                "one Llama-3-8B-shaped decoder layer (7 linear weights, 218,103,808 elems), B=1024"),
    4: Workload("llama3_8b_stack", (1024,), config4,
                "32 Llama-3-8B-shaped layers + embedding + LM head (226 tensors, "
                "8,029,995,008 elems, 16.06 GB BF16), B=1024"),
    5: Workload("mixed_specials_4096x14336", (128, 256, 512, 1024, 2048, 4096), config5,
                "BF16 4096x14336 N(0, 0.02) with a uniform-random 16-bit slab, a denormal slab "
                "and scattered +/-0, +/-Inf, NaN payloads, B in {128..4096}"),
}


def as_u16(t: torch.Tensor) -> torch.Tensor:
    """The BF16 tensor's bit patterns as int16 (same storage, no copy)."""
    return t.contiguous().view(torch.int16)
