"""CPU oracle for the WCB1 block fixed-length BF16 exponent code.

TEST INFRASTRUCTURE. Only ``tests/``, ``__graft_entry__.smoke()`` and the
``cpu_baseline`` / reference legs of ``bench.py`` may import this package. The
product library (``lossless_weight_compression_b200``) never imports it, and
the two share no code: the oracle is plain single-threaded C (``wc_oracle.c``)
written from the stream definition, wrapped here with ctypes.

Method source: "ENEC: A Lossless AI Model Compression Method Enabling Fast
Inference on Ascend NPUs", Abstract (per-block fixed-length code, bit-width
quantization, hierarchical halving packing, branch-free remap, prefix sum of
block sizes). Each wrapper below names the step of ``wc_oracle.c`` it calls.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "wc_oracle.c")
_LIB_PATH = os.path.join(_HERE, "liboracle.so")

OK, INVALID_ARG, BUFFER_TOO_SMALL, CORRUPT = 0, 1, 2, 3

_lib = None


def build(force: bool = False) -> str:
    """Compile ``wc_oracle.c`` into ``liboracle.so`` with gcc (plain C99, -O2)."""
    if (not force and os.path.exists(_LIB_PATH)
            and os.path.getmtime(_LIB_PATH) >= os.path.getmtime(_SRC)):
        return _LIB_PATH
    tmp = _LIB_PATH + ".tmp%d" % os.getpid()
    subprocess.run(["gcc", "-std=c99", "-O2", "-Wall", "-Wextra", "-fPIC", "-shared",
                    "-o", tmp, _SRC], check=True)
    os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def lib() -> ctypes.CDLL:
    global _lib
    if _lib is None:
        build()
        L = ctypes.CDLL(_LIB_PATH)
        u8, u16, u64, uint = ctypes.c_uint8, ctypes.c_uint16, ctypes.c_uint64, ctypes.c_uint
        vp = ctypes.c_void_p
        L.oracle_exponent.argtypes, L.oracle_exponent.restype = [u16], u8
        L.oracle_signman.argtypes, L.oracle_signman.restype = [u16], u8
        L.oracle_merge.argtypes, L.oracle_merge.restype = [u8, u8], u16
        L.oracle_bits.argtypes, L.oracle_bits.restype = [uint], uint
        L.oracle_block_params.argtypes = [vp, u64, vp, vp]
        L.oracle_block_params.restype = None
        L.oracle_pack_octet.argtypes, L.oracle_pack_octet.restype = [vp, uint], u64
        L.oracle_unpack_octet.argtypes = [u64, uint, vp]
        L.oracle_unpack_octet.restype = None
        L.oracle_bound.argtypes, L.oracle_bound.restype = [u64, ctypes.c_uint32], u64
        L.oracle_compress.argtypes = [vp, u64, ctypes.c_uint32, vp, u64, vp]
        L.oracle_compress.restype = ctypes.c_int
        L.oracle_decompress.argtypes = [vp, u64, vp, u64, ctypes.c_uint32]
        L.oracle_decompress.restype = ctypes.c_int
        L.oracle_bound_f32.argtypes, L.oracle_bound_f32.restype = [u64, ctypes.c_uint32], u64
        L.oracle_compress_f32.argtypes = [vp, u64, ctypes.c_uint32, vp, u64, vp]
        L.oracle_compress_f32.restype = ctypes.c_int
        L.oracle_decompress_f32.argtypes = [vp, u64, vp, u64, ctypes.c_uint32]
        L.oracle_decompress_f32.restype = ctypes.c_int
        L.oracle_esc_block_params.argtypes = [vp, u64, vp, vp, vp]
        L.oracle_esc_block_params.restype = None
        L.oracle_bound_escape.argtypes = [u64, ctypes.c_uint32]
        L.oracle_bound_escape.restype = u64
        L.oracle_compress_escape.argtypes = [vp, u64, ctypes.c_uint32, vp, u64, vp]
        L.oracle_compress_escape.restype = ctypes.c_int
        L.oracle_decompress_escape.argtypes = [vp, u64, vp, u64, ctypes.c_uint32]
        L.oracle_decompress_escape.restype = ctypes.c_int
        L.oracle_tans_normalize.argtypes = [vp, ctypes.c_uint32, vp]
        L.oracle_tans_normalize.restype = None
        L.oracle_tans_table.argtypes = [vp, ctypes.c_uint32, vp, vp, vp]
        L.oracle_tans_table.restype = None
        L.oracle_bound_tans.argtypes = [u64, ctypes.c_uint32, ctypes.c_uint32]
        L.oracle_bound_tans.restype = u64
        L.oracle_compress_tans.argtypes = [vp, u64, ctypes.c_uint32, ctypes.c_uint32, vp, u64, vp]
        L.oracle_compress_tans.restype = ctypes.c_int
        L.oracle_decompress_tans.argtypes = [vp, u64, vp, u64, ctypes.c_uint32]
        L.oracle_decompress_tans.restype = ctypes.c_int
        _lib = L
    return _lib


def _ptr(a: np.ndarray) -> int:
    return a.ctypes.data if a.size else 0


# --- step 1: split / merge -------------------------------------------------
def exponent(x: int) -> int:
    return lib().oracle_exponent(x)


def signman(x: int) -> int:
    return lib().oracle_signman(x)


def merge(e: int, s: int) -> int:
    return lib().oracle_merge(e, s)


# --- step 2: width quantization ----------------------------------------------
def bits(d: int) -> int:
    return lib().oracle_bits(d)


def block_params(words: np.ndarray) -> tuple[int, int]:
    """(base, w) of one block of BF16 bit patterns."""
    words = np.ascontiguousarray(words, dtype=np.uint16)
    base, w = ctypes.c_uint8(), ctypes.c_uint8()
    lib().oracle_block_params(_ptr(words), words.size, ctypes.byref(base), ctypes.byref(w))
    return base.value, w.value


# --- step 4: hierarchical halving pack ---------------------------------------
def pack_octet(values, w: int) -> int:
    v = np.ascontiguousarray(values, dtype=np.uint8)
    assert v.size == 8
    return lib().oracle_pack_octet(_ptr(v), w)


def unpack_octet(octet: int, w: int) -> list[int]:
    v = np.zeros(8, dtype=np.uint8)
    lib().oracle_unpack_octet(octet, w, _ptr(v))
    return v.tolist()


# --- whole streams -----------------------------------------------------------
def bound(n: int, block: int) -> int:
    return lib().oracle_bound(n, block)


def compress(words: np.ndarray, block: int) -> np.ndarray:
    """Encode BF16 bit patterns (uint16, any shape) into a WCB1 stream (uint8)."""
    words = np.ascontiguousarray(words, dtype=np.uint16).reshape(-1)
    cap = bound(words.size, block)
    if cap == 0:
        raise ValueError("oracle: invalid block size %r or n %d" % (block, words.size))
    out = np.empty(cap, dtype=np.uint8)
    nbytes = ctypes.c_uint64()
    rc = lib().oracle_compress(_ptr(words), words.size, block, _ptr(out), cap,
                               ctypes.byref(nbytes))
    if rc != OK:
        raise ValueError("oracle_compress failed with status %d" % rc)
    return out[: nbytes.value].copy()


def decompress_status(stream: np.ndarray, n: int, block: int) -> tuple[int, np.ndarray]:
    """Decode; returns (status, words). Status CORRUPT for any invalid stream."""
    stream = np.ascontiguousarray(stream, dtype=np.uint8).reshape(-1)
    out = np.zeros(n, dtype=np.uint16)
    rc = lib().oracle_decompress(_ptr(stream), stream.size, _ptr(out), n, block)
    return rc, out


def decompress(stream: np.ndarray, n: int, block: int) -> np.ndarray:
    rc, out = decompress_status(stream, n, block)
    if rc != OK:
        raise ValueError("oracle_decompress failed with status %d" % rc)
    return out


# --- FP32 streams: high halves coded as BF16 words, low halves raw ------------
def bound_f32(n: int, block: int) -> int:
    return lib().oracle_bound_f32(n, block)


def compress_f32(words: np.ndarray, block: int) -> np.ndarray:
    """Encode FP32 bit patterns (uint32, any shape) into an FP32 stream (uint8)."""
    words = np.ascontiguousarray(words, dtype=np.uint32).reshape(-1)
    cap = bound_f32(words.size, block)
    if cap == 0:
        raise ValueError("oracle: invalid block size %r or n %d" % (block, words.size))
    out = np.empty(cap, dtype=np.uint8)
    nbytes = ctypes.c_uint64()
    rc = lib().oracle_compress_f32(_ptr(words), words.size, block, _ptr(out), cap,
                                   ctypes.byref(nbytes))
    if rc != OK:
        raise ValueError("oracle_compress_f32 failed with status %d" % rc)
    return out[: nbytes.value].copy()


def decompress_f32_status(stream: np.ndarray, n: int, block: int) -> tuple[int, np.ndarray]:
    stream = np.ascontiguousarray(stream, dtype=np.uint8).reshape(-1)
    out = np.zeros(n, dtype=np.uint32)
    rc = lib().oracle_decompress_f32(_ptr(stream), stream.size, _ptr(out), n, block)
    return rc, out


def decompress_f32(stream: np.ndarray, n: int, block: int) -> np.ndarray:
    rc, out = decompress_f32_status(stream, n, block)
    if rc != OK:
        raise ValueError("oracle_decompress_f32 failed with status %d" % rc)
    return out


# --- fused decode + matrix-vector products (GEMV) -----------------------------
def bf16_to_f64(words: np.ndarray) -> np.ndarray:
    """BF16 bit patterns -> float64 values (a BF16 is the top half of an FP32)."""
    return (np.asarray(words, dtype=np.uint32) << 16).view(np.float32).astype(np.float64)


def gemv(stream: np.ndarray, rows: int, cols: int, block: int, x_words: np.ndarray):
    """y[j][r] = sum_c W[r][c] * x[j][c] in float64, W decoded from the stream by the
    C oracle; also returns sum_c |W[r][c] * x[j][c]| for the error bound. The
    definition written out: decode, then one float64 matrix product."""
    W = bf16_to_f64(decompress(stream, rows * cols, block)).reshape(rows, cols)
    x = bf16_to_f64(np.asarray(x_words, dtype=np.uint16).reshape(-1, cols))
    with np.errstate(invalid="ignore", over="ignore"):
        y = x @ W.T
        absum = np.abs(x) @ np.abs(W).T
    return y, absum


# --- escape-coded streams: a window of 2^w - 1 exponents + an exception list --
def esc_block_params(words: np.ndarray) -> tuple[int, int, int]:
    """(base, w, exceptions) of one block of an escape-coded stream."""
    words = np.ascontiguousarray(words, dtype=np.uint16)
    base, w, k = ctypes.c_uint8(), ctypes.c_uint8(), ctypes.c_uint64()
    lib().oracle_esc_block_params(_ptr(words), words.size, ctypes.byref(base),
                                  ctypes.byref(w), ctypes.byref(k))
    return base.value, w.value, k.value


def bound_escape(n: int, block: int) -> int:
    return lib().oracle_bound_escape(n, block)


def compress_escape(words: np.ndarray, block: int) -> np.ndarray:
    """Encode BF16 bit patterns (uint16, any shape) into an escape-coded stream."""
    words = np.ascontiguousarray(words, dtype=np.uint16).reshape(-1)
    cap = bound_escape(words.size, block)
    if cap == 0:
        raise ValueError("oracle: invalid block size %r or n %d" % (block, words.size))
    out = np.empty(cap, dtype=np.uint8)
    nbytes = ctypes.c_uint64()
    rc = lib().oracle_compress_escape(_ptr(words), words.size, block, _ptr(out), cap,
                                      ctypes.byref(nbytes))
    if rc != OK:
        raise ValueError("oracle_compress_escape failed with status %d" % rc)
    return out[: nbytes.value].copy()


def decompress_escape_status(stream: np.ndarray, n: int, block: int) -> tuple[int, np.ndarray]:
    stream = np.ascontiguousarray(stream, dtype=np.uint8).reshape(-1)
    out = np.zeros(n, dtype=np.uint16)
    rc = lib().oracle_decompress_escape(_ptr(stream), stream.size, _ptr(out), n, block)
    return rc, out


def decompress_escape(stream: np.ndarray, n: int, block: int) -> np.ndarray:
    rc, out = decompress_escape_status(stream, n, block)
    if rc != OK:
        raise ValueError("oracle_decompress_escape failed with status %d" % rc)
    return out


# --- tANS-coded streams: the exponents entropy-coded, 32 interleaved lanes ---
def tans_normalize(counts, R: int) -> np.ndarray:
    """Normalized counts (sum 2^R) of a 256-bin exponent histogram."""
    c = np.ascontiguousarray(counts, dtype=np.uint64)
    assert c.size == 256
    f = np.zeros(256, dtype=np.uint16)
    lib().oracle_tans_normalize(_ptr(c), R, _ptr(f))
    return f


def tans_table(freq, R: int):
    """(sym, nb, next) of every one of the 2^R decoder states."""
    f = np.ascontiguousarray(freq, dtype=np.uint16)
    L = 1 << R
    sym = np.zeros(L, np.uint8)
    nb = np.zeros(L, np.uint8)
    nxt = np.zeros(L, np.uint16)
    lib().oracle_tans_table(_ptr(f), R, _ptr(sym), _ptr(nb), _ptr(nxt))
    return sym, nb, nxt


def bound_tans(n: int, chunk: int, R: int) -> int:
    return lib().oracle_bound_tans(n, chunk, R)


def compress_tans(words: np.ndarray, chunk: int, R: int = 11) -> np.ndarray:
    """Encode BF16 bit patterns into a tANS-coded stream (chunk elements per
    chunk, 2^R table states)."""
    words = np.ascontiguousarray(words, dtype=np.uint16).reshape(-1)
    cap = bound_tans(words.size, chunk, R)
    if cap == 0:
        raise ValueError("oracle: invalid chunk %r, R %r or n %d" % (chunk, R, words.size))
    out = np.empty(cap, dtype=np.uint8)
    nbytes = ctypes.c_uint64()
    rc = lib().oracle_compress_tans(_ptr(words), words.size, chunk, R, _ptr(out), cap,
                                    ctypes.byref(nbytes))
    if rc != OK:
        raise ValueError("oracle_compress_tans failed with status %d" % rc)
    return out[: nbytes.value].copy()


def decompress_tans_status(stream: np.ndarray, n: int, chunk: int) -> tuple[int, np.ndarray]:
    stream = np.ascontiguousarray(stream, dtype=np.uint8).reshape(-1)
    out = np.zeros(n, dtype=np.uint16)
    rc = lib().oracle_decompress_tans(_ptr(stream), stream.size, _ptr(out), n, chunk)
    return rc, out


def decompress_tans(stream: np.ndarray, n: int, chunk: int) -> np.ndarray:
    rc, out = decompress_tans_status(stream, n, chunk)
    if rc != OK:
        raise ValueError("oracle_decompress_tans failed with status %d" % rc)
    return out
