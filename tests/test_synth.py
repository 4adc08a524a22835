"""The seeded synthetic inputs (the stand-ins for the pages' workloads) have the
shapes, value distributions and planted structure their recipe states, and are
the same on every call. CPU only; the stack itself (16 GB) is checked by its
element count and names, not generated."""
import numpy as np
import pytest
import torch

from lossless_weight_compression_b200 import synth


def u16(t):
    return t.contiguous().view(torch.int16).view(-1).numpy().view(np.uint16)


def test_config1_shape_distribution_and_determinism():
    (name, x), = synth.config1()
    assert x.shape == (1024, 1024) and x.dtype == torch.bfloat16
    assert abs(float(x.float().std()) - 0.02) < 0.0005
    assert abs(float(x.float().mean())) < 0.0005
    assert np.array_equal(u16(x), u16(synth.config1()[0][1]))


def test_config2_zero_rows_and_row_scales():
    (name, x), = synth.config2()
    assert x.shape == (4096, 4096) and x.dtype == torch.bfloat16
    xf = x.float()
    zero_rows = int((xf.abs().amax(dim=1) == 0).sum())
    assert zero_rows == 8
    assert not torch.any(torch.signbit(xf[xf.abs().amax(dim=1) == 0]))  # +0.0 rows
    # per-row scales spread over a decade: the 5th and 95th percentile of row
    # medians of |x| differ by far more than sampling noise
    med = xf.abs().median(dim=1).values
    med = med[med > 0]
    lo, hi = torch.quantile(med, 0.05).item(), torch.quantile(med, 0.95).item()
    assert hi / lo > 5.0
    # the planted +/-20 sigma outliers (16,777, ~4 per row): in almost every row
    # the largest |x| is far above the row's median
    ratio = xf.abs().amax(dim=1) / xf.abs().median(dim=1).values.clamp_min(1e-30)
    assert int((ratio > 15).sum()) > 3000


def test_layer_shapes_and_jittered_scales():
    shapes = [tuple(t.shape) for _, t in synth.layer_tensors(0)]
    assert shapes == [(r, c) for _, r, c in synth.LLAMA3_8B_LAYER]
    for name, t in synth.layer_tensors(0):
        s = float(t[:256].float().std())
        assert 0.02 * 0.69 < s < 0.02 * 1.31, name
    assert sum(r * c for _, r, c in synth.LLAMA3_8B_LAYER) == 218_103_808


def test_stack_size_and_names():
    names = synth.stack_names()
    assert len(names) == 226 and names[0] == "embed_tokens" and names[-1] == "lm_head"
    assert len(set(names)) == 226
    assert synth.STACK_ELEMS == 8_029_995_008
    assert 2 * synth.STACK_ELEMS == 16_059_990_016


def test_config5_slabs_and_specials():
    (name, x), = synth.config5()
    assert x.shape == synth.CFG5_SHAPE
    w = u16(x)
    exp = (w >> 7) & 0xFF
    # the denormal slab: exponent 0 with a nonzero mantissa, both signs, apart
    # from the few scattered specials that may land in it
    s, n = synth.CFG5_DENORMAL_SLAB
    slab = w[s:s + n]
    not_denormal = ((slab & 0x7F80) != 0) | ((slab & 0x7F) == 0)
    assert int(not_denormal.sum()) <= synth.CFG5_SPECIALS
    assert 0.45 < float((slab >> 15).mean()) < 0.55
    # the uniform-random slab holds every exponent, Inf/NaN ones included
    s, n = synth.CFG5_RANDOM_SLAB
    assert len(np.unique(exp[s:s + n])) == 256
    # outside the slabs the exponent range is that of N(0, 0.02) weights, plus specials
    rest = np.ones(w.size, bool)
    for s, n in (synth.CFG5_RANDOM_SLAB, synth.CFG5_DENORMAL_SLAB):
        rest[s:s + n] = False
    specials = np.isin(w, np.array(synth.SPECIAL_PATTERNS, np.uint16))
    assert int((specials & rest).sum()) > synth.CFG5_SPECIALS // 2
    gauss = rest & ~specials
    assert exp[gauss].max() < 127  # |x| < 1
    assert np.array_equal(w, u16(synth.config5()[0][1]))
