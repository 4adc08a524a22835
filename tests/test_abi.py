"""The C-ABI library on the host: it loads, exports every function that
include/wcodec.h declares, and its host-only arithmetic and argument checks
behave as documented. No call here launches a kernel (no GPU needed)."""
import ctypes
import os
import re

import numpy as np
import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
BLOCKS = (128, 256, 512, 1024, 2048, 4096)


def declared_functions():
    names = []
    for h in sorted(os.listdir(os.path.join(ROOT, "include"))):
        if not h.endswith(".h"):
            continue
        text = open(os.path.join(ROOT, "include", h)).read()
        text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)  # drop comments
        names += re.findall(r"^[A-Za-z_][\w \*]*?\b(wc_\w+)\s*\(", text, flags=re.M)
    return names


def test_header_declares_the_boundary():
    names = declared_functions()
    for f in ("wc_bound", "wc_workspace_size", "wc_compress", "wc_decompress",
              "wc_compress_batch", "wc_compress_batch_workspace_size",
              "wc_decompress_batch", "wc_stream_info", "wc_status_string", "wc_gemv",
              "wc_gemv_batch", "wc_gemm", "wc_gemm_batch",
              "wc_bound_fp32", "wc_compress_fp32", "wc_decompress_fp32",
              "wc_debug_compress_stalled"):
        assert f in names


def test_library_exports_every_declared_symbol(wclib):
    raw = ctypes.CDLL(wclib.LIB_PATH)
    for name in declared_functions():
        assert hasattr(raw, name), name


def test_bound_matches_oracle(wclib, orc):
    rng = np.random.default_rng(0)
    for B in BLOCKS:
        for n in [0, 1, 7, 8, 9, B - 1, B, B + 1, 8191, 8192, 8193] + list(rng.integers(0, 10**7, 5)):
            assert wclib.wc_bound(int(n), B) == orc.bound(int(n), B)
    for bad in (0, 1, 64, 127, 129, 384, 8192, 2**31):
        assert wclib.wc_bound(100, bad) == 0
    assert wclib.wc_bound(2**36, 1024) > 0 and wclib.wc_bound(2**36 + 1, 1024) == 0


def test_fp32_bound_matches_oracle(wclib, orc):
    rng = np.random.default_rng(1)
    for B in BLOCKS:
        for n in [0, 1, 7, 8, 9, B - 1, B, B + 1, 8193] + list(rng.integers(0, 10**7, 3)):
            assert wclib.wc_bound_fp32(int(n), B) == orc.bound_f32(int(n), B)
    assert wclib.wc_bound_fp32(100, 100) == 0


def test_stream_info_accepts_fp32_headers(wclib, orc):
    rng = np.random.default_rng(2)
    x = rng.integers(0, 2**32, 5000, dtype=np.uint64).astype(np.uint32)
    s = orc.compress_f32(x, 256)
    rc, n, block, total = wclib.wc_stream_info(s[:128].tobytes())
    assert (rc, n, block, total) == (0, 5000, 256, s.size)
    bad = s[:128].copy()
    bad[80] ^= 1  # the low plane's offset
    assert wclib.wc_stream_info(bad.tobytes())[0] == wclib.WC_ERR_CORRUPT_STREAM
    bad = s[:128].copy()
    bad[12] = 2  # unknown flag
    assert wclib.wc_stream_info(bad.tobytes())[0] == wclib.WC_ERR_CORRUPT_STREAM


def test_workspace_size(wclib):
    for n, tiles in [(0, 1), (1, 1), (8192, 1), (8193, 2), (10**6, 123)]:
        assert wclib.wc_workspace_size(n, 512) == 16 + 8 * tiles
    assert wclib.wc_workspace_size(10, 100) == 0


def test_stream_info_parses_oracle_headers(wclib, orc):
    rng = np.random.default_rng(1)
    for B in BLOCKS:
        for n in (0, 1, 1000, 3 * B + 5):
            words = rng.integers(0, 65536, n).astype(np.uint16)
            s = orc.compress(words, B)
            rc, nn, bb, tot = wclib.wc_stream_info(bytes(s[:128]))
            assert (rc, nn, bb, tot) == (0, n, B, s.size)


def test_stream_info_rejects_bad_headers(wclib, orc):
    s = orc.compress(np.arange(5000, dtype=np.uint16), 256)
    good = bytes(s[:128])
    assert wclib.wc_stream_info(good)[0] == wclib.WC_OK
    for off, val in [(0, 0), (4, 2), (6, 64), (8, 0x7F), (12, 1), (16, 0x99), (24, 3), (40, 1),
                     (64, 0xFF), (72, 0), (100, 1)]:
        b = bytearray(good)
        b[off] = (b[off] + val) & 0xFF if val else (b[off] ^ 0xFF)
        assert wclib.wc_stream_info(bytes(b))[0] == wclib.WC_ERR_CORRUPT_STREAM, off
    assert wclib.wc_stream_info(good[:64])[0] == wclib.WC_ERR_INVALID_ARG


def test_status_strings(wclib):
    for code in range(6):
        assert wclib.wc_status_string(code)
    assert wclib.wc_status_string(99) == "unknown status"


def test_argument_checks_before_any_launch(wclib):
    """Invalid arguments are rejected on the host; these calls never reach CUDA."""
    c = wclib
    # null input with n > 0, null output, invalid block, misaligned pointers
    assert c.wc_compress(None, 10, 128, 16, 10**6, 16, 16, 10**6, None, None) == c.WC_ERR_INVALID_ARG
    assert c.wc_compress(16, 10, 128, None, 10**6, 16, 16, 10**6, None, None) == c.WC_ERR_INVALID_ARG
    assert c.wc_compress(16, 10, 100, 16, 10**6, 16, 16, 10**6, None, None) == c.WC_ERR_INVALID_ARG
    assert c.wc_compress(17, 10, 128, 16, 10**6, 16, 16, 10**6, None, None) == c.WC_ERR_INVALID_ARG
    assert c.wc_compress(16, 10, 128, 16, 10, 16, 16, 10**6, None, None) == c.WC_ERR_BUFFER_TOO_SMALL
    assert c.wc_compress(16, 10, 128, 16, 10**6, 16, 16, 8, None, None) == c.WC_ERR_BUFFER_TOO_SMALL
    # decode: stream shorter than the fixed sections, null stream, misaligned output, bad block
    assert c.wc_decompress(16, 100, 16, 10, 128, None, None) == c.WC_ERR_CORRUPT_STREAM
    assert c.wc_decompress(None, 10**6, 16, 10, 128, None, None) == c.WC_ERR_INVALID_ARG
    assert c.wc_decompress(16, 10**6, 18, 10, 128, None, None) == c.WC_ERR_INVALID_ARG
    assert c.wc_decompress(16, 10**6, 16, 10, 3000, None, None) == c.WC_ERR_INVALID_ARG
    # batch: every item is checked before anything is launched
    arr, count = c.make_batch([])
    items = (c.wc_batch_item * 2)()
    items[0].stream, items[0].stream_bytes, items[0].out, items[0].n, items[0].block = 16, 10**6, 16, 10, 128
    items[1].stream, items[1].stream_bytes, items[1].out, items[1].n, items[1].block = 16, 10**6, 16, 10, 99
    assert c.wc_decompress_batch(items, 2, None, None) == c.WC_ERR_INVALID_ARG
    items[1].block, items[1].reserved = 128, 1
    assert c.wc_decompress_batch(items, 2, None, None) == c.WC_ERR_INVALID_ARG
    assert c.wc_decompress_batch(None, 1, None, None) == c.WC_ERR_INVALID_ARG
    # batched compression: every item is checked before anything is launched
    citems = (c.wc_compress_item * 2)()
    for j in range(2):
        citems[j].in_, citems[j].n, citems[j].block = 16, 10, 128
        citems[j].out, citems[j].out_capacity, citems[j].out_bytes = 16, 10**6, 16
    citems[1].block = 100
    assert c.wc_compress_batch(citems, 2, 16, 10**6, None, None) == c.WC_ERR_INVALID_ARG
    assert c.wc_compress_batch_workspace_size(citems, 2) == 0
    citems[1].block, citems[1].reserved = 128, 7
    assert c.wc_compress_batch(citems, 2, 16, 10**6, None, None) == c.WC_ERR_INVALID_ARG
    citems[1].reserved = 0
    assert c.wc_compress_batch_workspace_size(citems, 2) == 2 * 8 + 16
    assert c.wc_compress_batch(citems, 2, 16, 8, None, None) == c.WC_ERR_BUFFER_TOO_SMALL
    citems[1].out_capacity = 10
    assert c.wc_compress_batch(citems, 2, 16, 10**6, None, None) == c.WC_ERR_BUFFER_TOO_SMALL
    # fused decode-GEMV: shapes and vector counts are checked on the host
    assert c.wc_gemv(16, 10**6, 4, 1000, 128, 16, 1, 16, None, None) == c.WC_ERR_INVALID_ARG  # cols % B
    assert c.wc_gemv(16, 10**6, 4, 1024, 128, 16, 3, 16, None, None) == c.WC_ERR_INVALID_ARG  # n_vec
    assert c.wc_gemv(16, 10**6, 4, 1024, 128, 17, 1, 16, None, None) == c.WC_ERR_INVALID_ARG  # x align
    assert c.wc_gemv(16, 100, 4, 1024, 128, 16, 1, 16, None, None) == c.WC_ERR_CORRUPT_STREAM
    # FP32 streams: capacity and truncation are checked on the host
    assert c.wc_compress_fp32(16, 1000, 128, 16, 100, 16, 16, 10**6, None, None) == \
        c.WC_ERR_BUFFER_TOO_SMALL
    assert c.wc_compress_fp32(16, 1000, 100, 16, 10**6, 16, 16, 10**6, None, None) == \
        c.WC_ERR_INVALID_ARG
    assert c.wc_decompress_fp32(16, 100, 16, 1000, 128, None, None) == c.WC_ERR_CORRUPT_STREAM
    assert c.wc_decompress_fp32(16, 10**6, 16, 1000, 100, None, None) == c.WC_ERR_INVALID_ARG
    # fused decode-GEMM on the tensor cores: token count, cols % 128, alignment, truncation
    assert c.wc_gemm(16, 10**6, 4, 1024, 128, 16, 0, 16, None, None) == c.WC_ERR_INVALID_ARG
    assert c.wc_gemm(16, 10**6, 4, 1024, 128, 16, 129, 16, None, None) == c.WC_ERR_INVALID_ARG
    assert c.wc_gemm(16, 10**6, 4, 1000, 128, 16, 16, 16, None, None) == c.WC_ERR_INVALID_ARG
    assert c.wc_gemm(16, 10**6, 4, 1024, 100, 16, 16, 16, None, None) == c.WC_ERR_INVALID_ARG
    assert c.wc_gemm(16, 10**6, 4, 1024, 128, 24, 16, 16, None, None) == c.WC_ERR_INVALID_ARG
    assert c.wc_gemm(24, 10**6, 4, 1024, 128, 16, 16, 16, None, None) == c.WC_ERR_INVALID_ARG
    assert c.wc_gemm(16, 10**6, 4, 1024, 128, 16, 16, 18, None, None) == c.WC_ERR_INVALID_ARG
    assert c.wc_gemm(16, 100, 4, 1024, 128, 16, 16, 16, None, None) == c.WC_ERR_CORRUPT_STREAM
    gitems = (c.wc_gemv_item * 2)()
    for it in gitems:
        it.stream, it.stream_bytes, it.x, it.y = 16, 10**6, 16, 16
        it.rows, it.cols, it.block, it.reserved = 4, 1024, 128, 0
    gitems[1].reserved = 1
    assert c.wc_gemm_batch(gitems, 2, 16, None, None) == c.WC_ERR_INVALID_ARG
    assert c.wc_gemm_batch(None, 1, 16, None, None) == c.WC_ERR_INVALID_ARG
    # the stall test hook needs two tiles and a bounded timeout
    assert c.wc_debug_compress_stalled(16, 100, 128, 16, 10**6, 16, 16, 10**6, None, 10**6,
                                       None) == c.WC_ERR_INVALID_ARG
    assert c.wc_debug_compress_stalled(16, 10**5, 128, 16, 10**7, 16, 16, 10**6, None, 0,
                                       None) == c.WC_ERR_INVALID_ARG


def test_binding_fails_loudly_without_the_library(monkeypatch, tmp_path):
    from lossless_weight_compression_b200 import wcodec
    monkeypatch.setattr(wcodec, "_lib", None)
    monkeypatch.setattr(wcodec, "LIB_PATH", str(tmp_path / "missing.so"))
    with pytest.raises(RuntimeError, match="not built"):
        wcodec.lib()


def test_escape_bound_matches_oracle(wclib, orc):
    rng = np.random.default_rng(2)
    for B in BLOCKS:
        for n in [0, 1, 7, 8, 9, B - 1, B, B + 1, 8193] + list(rng.integers(0, 10**7, 3)):
            assert wclib.wc_bound_escape(int(n), B) == orc.bound_escape(int(n), B)
            assert wclib.wc_workspace_size_escape(int(n), B) >= 16
    assert wclib.wc_bound_escape(100, 100) == 0 and wclib.wc_workspace_size_escape(100, 100) == 0


def test_escape_entry_points_check_arguments_before_launching(wclib):
    # fake, aligned device addresses: every call below must return before any launch
    n, B = 10_000, 1024
    cap, ws = wclib.wc_bound_escape(n, B), wclib.wc_workspace_size_escape(n, B)
    rc = wclib.wc_compress_escape(1 << 20, n, 1000, 1 << 21, cap, 1 << 22, 1 << 23, ws, None, None)
    assert rc == wclib.WC_ERR_INVALID_ARG                   # block size
    rc = wclib.wc_compress_escape(1 << 20, n, B, (1 << 21) + 8, cap, 1 << 22, 1 << 23, ws, None, None)
    assert rc == wclib.WC_ERR_INVALID_ARG                   # misaligned output
    rc = wclib.wc_compress_escape(1 << 20, n, B, 1 << 21, cap - 1, 1 << 22, 1 << 23, ws, None, None)
    assert rc == wclib.WC_ERR_BUFFER_TOO_SMALL              # output capacity
    rc = wclib.wc_compress_escape(1 << 20, n, B, 1 << 21, cap, 1 << 22, 1 << 23, ws - 1, None, None)
    assert rc == wclib.WC_ERR_BUFFER_TOO_SMALL              # workspace
    rc = wclib.wc_decompress_escape(1 << 20, 100, 1 << 21, n, B, None, None)
    assert rc == wclib.WC_ERR_CORRUPT_STREAM                # shorter than the fixed sections
    rc = wclib.wc_decompress_escape_batch(None, 3, None, None)
    assert rc == wclib.WC_ERR_INVALID_ARG


def test_stream_info_reads_escape_headers(wclib, orc):
    words = (np.random.default_rng(3).standard_normal(5000) * 0.02).astype(np.float32)
    words = (words.view(np.uint32) >> 16).astype(np.uint16)
    s = orc.compress_escape(words, 256)
    rc, n, b, total = wclib.wc_stream_info(bytes(s[:128]))
    assert rc == wclib.WC_OK and (n, b, total) == (5000, 256, s.size)


def test_host_stream_decode_checks_flags_before_anything(wclib):
    item = (wclib.wc_batch_item * 1)()
    for bad_flags in (1, 3, 4):
        assert wclib.wc_decompress_host_batch(item, 1, bad_flags, None, None) == wclib.WC_ERR_INVALID_ARG
    assert wclib.wc_decompress_host_batch(None, 2, 0, None, None) == wclib.WC_ERR_INVALID_ARG
