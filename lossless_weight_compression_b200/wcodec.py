"""ctypes binding of libwcodec (include/wcodec.h), plus torch-tensor helpers.

The ``wc_*`` functions take the same arguments as the C functions (device
pointers as ints, sizes, a cudaStream_t as an int); they only marshal
arguments. Every step of compression and decompression runs in the library's
CUDA kernels; there is no Python or CPU fallback, and loading fails loudly if
``libwcodec.so`` has not been built (``python -m
lossless_weight_compression_b200.build_lib``).

The helpers below (``compress``, ``decompress``, ...) take torch tensors,
allocate outputs with torch and call the same entry points.
"""
from __future__ import annotations

import ctypes
import os
from dataclasses import dataclass

import torch

LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libwcodec.so")

WC_OK = 0
WC_ERR_INVALID_ARG = 1
WC_ERR_BUFFER_TOO_SMALL = 2
WC_ERR_CORRUPT_STREAM = 3
WC_ERR_CUDA = 4
WC_ERR_TIMEOUT = 5
WC_HEADER_BYTES = 128
WC_BATCH_MAX = 512
BLOCK_SIZES = (128, 256, 512, 1024, 2048, 4096)


class WcodecError(RuntimeError):
    def __init__(self, status: int, what: str):
        super().__init__("%s: %s (status %d)" % (what, wc_status_string(status), status))
        self.status = status


class wc_compress_item(ctypes.Structure):
    _fields_ = [
        ("in_", ctypes.c_void_p),
        ("n", ctypes.c_uint64),
        ("block", ctypes.c_uint32),
        ("reserved", ctypes.c_uint32),
        ("out", ctypes.c_void_p),
        ("out_capacity", ctypes.c_uint64),
        ("out_bytes", ctypes.c_void_p),
    ]


class wc_gemv_item(ctypes.Structure):
    _fields_ = [
        ("stream", ctypes.c_void_p),
        ("stream_bytes", ctypes.c_uint64),
        ("x", ctypes.c_void_p),
        ("y", ctypes.c_void_p),
        ("rows", ctypes.c_uint32),
        ("cols", ctypes.c_uint32),
        ("block", ctypes.c_uint32),
        ("reserved", ctypes.c_uint32),
    ]


class wc_batch_item(ctypes.Structure):
    _fields_ = [
        ("stream", ctypes.c_void_p),
        ("stream_bytes", ctypes.c_uint64),
        ("out", ctypes.c_void_p),
        ("n", ctypes.c_uint64),
        ("block", ctypes.c_uint32),
        ("reserved", ctypes.c_uint32),
    ]


_lib = None


def lib() -> ctypes.CDLL:
    """Load libwcodec.so (once). Raises if it is missing: there is no fallback."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise RuntimeError(
            "libwcodec.so is not built (%s); run `python -m lossless_weight_compression_b200."
            "build_lib`" % LIB_PATH)
    L = ctypes.CDLL(LIB_PATH)
    u32, u64, vp, i = ctypes.c_uint32, ctypes.c_uint64, ctypes.c_void_p, ctypes.c_int
    L.wc_bound.argtypes, L.wc_bound.restype = [u64, u32], u64
    L.wc_workspace_size.argtypes, L.wc_workspace_size.restype = [u64, u32], u64
    L.wc_compress.argtypes = [vp, u64, u32, vp, u64, vp, vp, u64, vp, vp]
    L.wc_compress.restype = i
    L.wc_decompress.argtypes = [vp, u64, vp, u64, u32, vp, vp]
    L.wc_decompress.restype = i
    L.wc_decompress_batch.argtypes = [ctypes.POINTER(wc_batch_item), u32, vp, vp]
    L.wc_decompress_batch.restype = i
    L.wc_stream_info.argtypes = [vp, u64, ctypes.POINTER(u64), ctypes.POINTER(u32),
                                 ctypes.POINTER(u64)]
    L.wc_stream_info.restype = i
    L.wc_status_string.argtypes, L.wc_status_string.restype = [i], ctypes.c_char_p
    L.wc_compress_batch_workspace_size.argtypes = [ctypes.POINTER(wc_compress_item), u32]
    L.wc_compress_batch_workspace_size.restype = u64
    L.wc_compress_batch.argtypes = [ctypes.POINTER(wc_compress_item), u32, vp, u64, vp, vp]
    L.wc_compress_batch.restype = i
    L.wc_gemv.argtypes = [vp, u64, u32, u32, u32, vp, u32, vp, vp, vp]
    L.wc_gemv.restype = i
    L.wc_gemv_batch.argtypes = [ctypes.POINTER(wc_gemv_item), u32, u32, vp, vp]
    L.wc_gemv_batch.restype = i
    L.wc_bound_fp32.argtypes, L.wc_bound_fp32.restype = [u64, u32], u64
    L.wc_compress_fp32.argtypes = [vp, u64, u32, vp, u64, vp, vp, u64, vp, vp]
    L.wc_compress_fp32.restype = i
    L.wc_decompress_fp32.argtypes = [vp, u64, vp, u64, u32, vp, vp]
    L.wc_decompress_fp32.restype = i
    L.wc_gemm.argtypes = [vp, u64, u32, u32, u32, vp, u32, vp, vp, vp]
    L.wc_gemm.restype = i
    L.wc_gemm_batch.argtypes = [ctypes.POINTER(wc_gemv_item), u32, u32, vp, vp]
    L.wc_gemm_batch.restype = i
    L.wc_gemm_batch_flags.argtypes = [ctypes.POINTER(wc_gemv_item), u32, u32, u32, vp, vp]
    L.wc_gemm_batch_flags.restype = i
    L.wc_bound_tans.argtypes, L.wc_bound_tans.restype = [u64, u32, u32], u64
    L.wc_compress_tans_batch_workspace_size.argtypes = [ctypes.POINTER(wc_compress_item), u32]
    L.wc_compress_tans_batch_workspace_size.restype = u64
    L.wc_compress_tans.argtypes = [vp, u64, u32, u32, vp, u64, vp, vp, u64, vp]
    L.wc_compress_tans.restype = i
    L.wc_compress_tans_batch.argtypes = [ctypes.POINTER(wc_compress_item), u32, u32, vp, u64, vp]
    L.wc_compress_tans_batch.restype = i
    L.wc_decompress_tans.argtypes = [vp, u64, vp, u64, u32, vp, vp]
    L.wc_decompress_tans.restype = i
    L.wc_decompress_tans_batch.argtypes = [ctypes.POINTER(wc_batch_item), u32, vp, vp]
    L.wc_decompress_tans_batch.restype = i
    L.wc_compress_noalloc.argtypes = [vp, u64, u32, vp, u64, vp, vp, vp]
    L.wc_compress_noalloc.restype = i
    L.wc_debug_compress_stalled.argtypes = [vp, u64, u32, vp, u64, vp, vp, u64, vp, u64, vp]
    L.wc_debug_compress_stalled.restype = i
    L.wc_bound_escape.argtypes, L.wc_bound_escape.restype = [u64, u32], u64
    L.wc_workspace_size_escape.argtypes, L.wc_workspace_size_escape.restype = [u64, u32], u64
    L.wc_compress_escape.argtypes = [vp, u64, u32, vp, u64, vp, vp, u64, vp, vp]
    L.wc_compress_escape.restype = i
    L.wc_decompress_escape.argtypes = [vp, u64, vp, u64, u32, vp, vp]
    L.wc_decompress_escape.restype = i
    L.wc_decompress_escape_batch.argtypes = [ctypes.POINTER(wc_batch_item), u32, vp, vp]
    L.wc_decompress_escape_batch.restype = i
    L.wc_compress_escape_batch_workspace_size.argtypes = [ctypes.POINTER(wc_compress_item), u32]
    L.wc_compress_escape_batch_workspace_size.restype = u64
    L.wc_compress_escape_batch.argtypes = [ctypes.POINTER(wc_compress_item), u32, vp, u64, vp, vp]
    L.wc_compress_escape_batch.restype = i
    L.wc_decompress_host.argtypes = [vp, u64, vp, u64, u32, u32, vp, vp]
    L.wc_decompress_host.restype = i
    L.wc_decompress_host_batch.argtypes = [ctypes.POINTER(wc_batch_item), u32, u32, vp, vp]
    L.wc_decompress_host_batch.restype = i
    _lib = L
    return L


# ---------------------------------------------------------------------------
# The C functions, same names and arguments
# ---------------------------------------------------------------------------
def wc_bound(n: int, block: int) -> int:
    return lib().wc_bound(n, block)


def wc_workspace_size(n: int, block: int) -> int:
    return lib().wc_workspace_size(n, block)


def wc_compress(d_in, n, block, d_out, out_capacity, d_out_bytes, d_workspace, workspace_bytes,
                d_status, stream) -> int:
    return lib().wc_compress(d_in, n, block, d_out, out_capacity, d_out_bytes, d_workspace,
                             workspace_bytes, d_status, stream)


def wc_compress_batch_workspace_size(items, count) -> int:
    return lib().wc_compress_batch_workspace_size(items, count)


def wc_compress_batch(items, count, d_workspace, workspace_bytes, d_status, stream) -> int:
    return lib().wc_compress_batch(items, count, d_workspace, workspace_bytes, d_status, stream)


def wc_compress_noalloc(d_in, n, block, d_out, out_capacity, d_out_bytes, d_status,
                        stream) -> int:
    """wc_compress without a workspace, for callers that cannot allocate device
    memory; its scratch is a fixed array in the library (n <= 2^30)."""
    return lib().wc_compress_noalloc(d_in, n, block, d_out, out_capacity, d_out_bytes, d_status,
                                     stream)


def wc_decompress(d_stream, stream_bytes, d_out, n, block, d_status, stream) -> int:
    return lib().wc_decompress(d_stream, stream_bytes, d_out, n, block, d_status, stream)


def wc_decompress_batch(items, count, d_status, stream) -> int:
    return lib().wc_decompress_batch(items, count, d_status, stream)


def wc_gemv(d_stream, stream_bytes, rows, cols, block, d_x, n_vec, d_y, d_status, stream) -> int:
    return lib().wc_gemv(d_stream, stream_bytes, rows, cols, block, d_x, n_vec, d_y, d_status,
                         stream)


def wc_gemv_batch(items, count, n_vec, d_status, stream) -> int:
    return lib().wc_gemv_batch(items, count, n_vec, d_status, stream)


def wc_bound_fp32(n, block) -> int:
    return lib().wc_bound_fp32(n, block)


def wc_compress_fp32(d_in, n, block, d_out, out_capacity, d_out_bytes, d_ws, ws_bytes, d_status,
                     stream) -> int:
    return lib().wc_compress_fp32(d_in, n, block, d_out, out_capacity, d_out_bytes, d_ws,
                                  ws_bytes, d_status, stream)


def wc_decompress_fp32(d_stream, stream_bytes, d_out, n, block, d_status, stream) -> int:
    return lib().wc_decompress_fp32(d_stream, stream_bytes, d_out, n, block, d_status, stream)


def wc_gemm(d_stream, stream_bytes, rows, cols, block, d_x, tokens, d_y, d_status, stream) -> int:
    return lib().wc_gemm(d_stream, stream_bytes, rows, cols, block, d_x, tokens, d_y, d_status,
                         stream)


def wc_bound_tans(n, chunk, table_log) -> int:
    return lib().wc_bound_tans(n, chunk, table_log)


def wc_compress_tans_batch_workspace_size(items, count) -> int:
    return lib().wc_compress_tans_batch_workspace_size(items, count)


def wc_compress_tans(d_in, n, chunk, table_log, d_out, out_capacity, d_out_bytes, d_ws, ws_bytes,
                     stream) -> int:
    return lib().wc_compress_tans(d_in, n, chunk, table_log, d_out, out_capacity, d_out_bytes,
                                  d_ws, ws_bytes, stream)


def wc_compress_tans_batch(items, count, table_log, d_ws, ws_bytes, stream) -> int:
    return lib().wc_compress_tans_batch(items, count, table_log, d_ws, ws_bytes, stream)


def wc_decompress_tans(d_stream, stream_bytes, d_out, n, chunk, d_status, stream) -> int:
    return lib().wc_decompress_tans(d_stream, stream_bytes, d_out, n, chunk, d_status, stream)


def wc_decompress_tans_batch(items, count, d_status, stream) -> int:
    return lib().wc_decompress_tans_batch(items, count, d_status, stream)


def wc_gemm_batch_flags(items, count, tokens, flags, d_status, stream) -> int:
    return lib().wc_gemm_batch_flags(items, count, tokens, flags, d_status, stream)


def wc_gemm_batch(items, count, tokens, d_status, stream) -> int:
    return lib().wc_gemm_batch(items, count, tokens, d_status, stream)


def wc_bound_escape(n, block) -> int:
    return lib().wc_bound_escape(n, block)


def wc_workspace_size_escape(n, block) -> int:
    return lib().wc_workspace_size_escape(n, block)


def wc_compress_escape(d_in, n, block, d_out, out_capacity, d_out_bytes, d_ws, ws_bytes, d_status,
                       stream) -> int:
    return lib().wc_compress_escape(d_in, n, block, d_out, out_capacity, d_out_bytes, d_ws,
                                    ws_bytes, d_status, stream)


def wc_decompress_escape(d_stream, stream_bytes, d_out, n, block, d_status, stream) -> int:
    return lib().wc_decompress_escape(d_stream, stream_bytes, d_out, n, block, d_status, stream)


def wc_decompress_escape_batch(items, count, d_status, stream) -> int:
    return lib().wc_decompress_escape_batch(items, count, d_status, stream)


WC_FLAG_ESCAPE = 2


def wc_compress_escape_batch_workspace_size(items, count) -> int:
    return lib().wc_compress_escape_batch_workspace_size(items, count)


def wc_compress_escape_batch(items, count, d_workspace, workspace_bytes, d_status, stream) -> int:
    return lib().wc_compress_escape_batch(items, count, d_workspace, workspace_bytes, d_status,
                                          stream)


def wc_decompress_host(h_stream, stream_bytes, d_out, n, block, flags, d_status, stream) -> int:
    return lib().wc_decompress_host(h_stream, stream_bytes, d_out, n, block, flags, d_status,
                                    stream)


def wc_decompress_host_batch(items, count, flags, d_status, stream) -> int:
    return lib().wc_decompress_host_batch(items, count, flags, d_status, stream)


def wc_stream_info(h_header: bytes):
    """Returns (status, n, block, total_bytes) parsed from a host copy of the header."""
    n, blk, tot = ctypes.c_uint64(), ctypes.c_uint32(), ctypes.c_uint64()
    buf = ctypes.create_string_buffer(bytes(h_header), len(h_header))
    rc = lib().wc_stream_info(ctypes.cast(buf, ctypes.c_void_p), len(h_header), ctypes.byref(n),
                              ctypes.byref(blk), ctypes.byref(tot))
    return rc, n.value, blk.value, tot.value


def wc_status_string(status: int) -> str:
    return lib().wc_status_string(status).decode()


def wc_debug_compress_stalled(d_in, n, block, d_out, out_capacity, d_out_bytes, d_workspace,
                              workspace_bytes, d_status, timeout_ns, stream) -> int:
    return lib().wc_debug_compress_stalled(d_in, n, block, d_out, out_capacity, d_out_bytes,
                                           d_workspace, workspace_bytes, d_status, timeout_ns,
                                           stream)


# ---------------------------------------------------------------------------
# torch helpers
# ---------------------------------------------------------------------------
def _stream_handle(stream) -> int:
    s = stream if stream is not None else torch.cuda.current_stream()
    return s.cuda_stream


def _check(rc: int, what: str):
    if rc != WC_OK:
        raise WcodecError(rc, what)


def as_words(x: torch.Tensor) -> torch.Tensor:
    """A 16-bit tensor (bf16 / int16 / uint16 / fp16) as contiguous flat int16 words."""
    if x.element_size() != 2:
        raise TypeError("wcodec compresses 16-bit words (BF16); got %s" % x.dtype)
    return x.contiguous().view(-1).view(torch.int16)


@dataclass
class Compressed:
    """A compressed tensor on the GPU: ``buffer`` holds ``wc_bound`` bytes of
    which the first ``nbytes`` (a device int64) are the stream."""
    buffer: torch.Tensor
    nbytes: torch.Tensor
    status: torch.Tensor
    n: int
    block: int
    shape: tuple
    dtype: torch.dtype
    escape: bool = False  # an escape-coded stream (header flags bit 1)

    def size(self) -> int:
        return int(self.nbytes.item())

    def stream(self) -> torch.Tensor:
        """The stream bytes (synchronises to read the size)."""
        return self.buffer[: self.size()]


def workspace_for(n: int, block: int, device) -> torch.Tensor:
    ws = wc_workspace_size(n, block)
    if ws == 0:
        raise WcodecError(WC_ERR_INVALID_ARG, "workspace size")
    return torch.empty((ws + 15) // 16 * 16, dtype=torch.uint8, device=device)


def compress(x: torch.Tensor, block: int = 1024, *, workspace: torch.Tensor | None = None,
             stream=None) -> Compressed:
    """Compress a CUDA tensor of BF16 (any 16-bit dtype is read as bit patterns)."""
    words = as_words(x)
    n = words.numel()
    cap = wc_bound(n, block)
    if cap == 0:
        raise WcodecError(WC_ERR_INVALID_ARG, "block size %r" % (block,))
    dev = words.device
    buf = torch.empty((cap + 15) // 16 * 16, dtype=torch.uint8, device=dev)
    nbytes = torch.zeros(1, dtype=torch.int64, device=dev)
    status = torch.zeros(1, dtype=torch.int32, device=dev)
    if workspace is None:
        workspace = workspace_for(n, block, dev)
    rc = wc_compress(words.data_ptr() if n else None, n, block, buf.data_ptr(), buf.numel(),
                     nbytes.data_ptr(), workspace.data_ptr(), workspace.numel(),
                     status.data_ptr(), _stream_handle(stream))
    _check(rc, "wc_compress")
    return Compressed(buf, nbytes, status, n, block, tuple(x.shape), x.dtype)


def decompress(stream_bytes: torch.Tensor, n: int, block: int, *, out: torch.Tensor | None = None,
               status: torch.Tensor | None = None, nbytes: int | None = None,
               stream=None) -> torch.Tensor:
    """Decode a stream (a uint8 CUDA tensor) into n BF16 values (``out`` if given)."""
    if out is None:
        out = torch.empty(n, dtype=torch.bfloat16, device=stream_bytes.device)
    words = out.view(-1)
    if words.numel() != n or not words.is_contiguous() or out.element_size() != 2:
        raise ValueError("out must be a contiguous 16-bit tensor of %d elements" % n)
    own_status = status is None
    if own_status:
        status = torch.zeros(1, dtype=torch.int32, device=stream_bytes.device)
    size = stream_bytes.numel() if nbytes is None else nbytes
    rc = wc_decompress(stream_bytes.data_ptr(), size, words.data_ptr() if n else None, n, block,
                       status.data_ptr(), _stream_handle(stream))
    _check(rc, "wc_decompress")
    return out


def decompress_compressed(c: Compressed, out: torch.Tensor | None = None, status=None,
                          stream=None) -> torch.Tensor:
    """Decode a ``Compressed`` (plain or escape-coded) back into its original shape and dtype."""
    if out is None:
        out = torch.empty(c.shape, dtype=c.dtype, device=c.buffer.device)
    fn = decompress_escape if c.escape else decompress
    return fn(c.buffer, c.n, c.block, out=out, status=status, stream=stream)


class CompressBatch:
    """Reusable buffers and descriptors for compressing a fixed list of tensors
    in one call: ``run()`` enqueues one encoder launch per 512 tensors (five for
    escape-coded streams, ``escape=True``; five per 512 for tANS-coded streams,
    ``tans_log=R``, whose ``block`` is then the chunk size)."""

    def __init__(self, tensors, block=1024, escape=False, tans_log=None):
        self.escape = escape
        self.tans_log = tans_log
        if tans_log is not None:
            def bound(n, b):
                return wc_bound_tans(n, b, tans_log)
        else:
            bound = wc_bound_escape if escape else wc_bound
        self.words = [as_words(t) for t in tensors]
        dev = self.words[0].device if self.words else torch.device("cuda")
        k = len(self.words)
        self.blocks = list(block) if isinstance(block, (list, tuple)) else [block] * k
        self.buffers = [torch.empty((bound(w.numel(), b) + 15) // 16 * 16,
                                    dtype=torch.uint8, device=dev)
                        for w, b in zip(self.words, self.blocks)]
        self.nbytes = torch.zeros(max(1, k), dtype=torch.int64, device=dev)
        self.status = torch.zeros(1, dtype=torch.int32, device=dev)
        self.items = (wc_compress_item * max(1, k))()
        for j, w in enumerate(self.words):
            it = self.items[j]
            it.in_ = w.data_ptr() if w.numel() else None
            it.n = w.numel()
            it.block = self.blocks[j]
            it.reserved = 0
            it.out = self.buffers[j].data_ptr()
            it.out_capacity = self.buffers[j].numel()
            it.out_bytes = self.nbytes[j:].data_ptr()
        if tans_log is not None:
            ws = wc_compress_tans_batch_workspace_size(self.items, k)
        else:
            ws = (wc_compress_escape_batch_workspace_size if escape
                  else wc_compress_batch_workspace_size)(self.items, k)
        if k and ws == 0:
            raise WcodecError(WC_ERR_INVALID_ARG, "workspace size")
        self.workspace = torch.empty(max(16, (ws + 15) // 16 * 16), dtype=torch.uint8, device=dev)
        self.count = k

    def run(self, stream=None):
        if self.tans_log is not None:
            rc = wc_compress_tans_batch(self.items, self.count, self.tans_log,
                                        self.workspace.data_ptr(), self.workspace.numel(),
                                        _stream_handle(stream))
            _check(rc, "wc_compress_tans_batch")
            return
        entry = wc_compress_escape_batch if self.escape else wc_compress_batch
        rc = entry(self.items, self.count, self.workspace.data_ptr(), self.workspace.numel(),
                   self.status.data_ptr(), _stream_handle(stream))
        _check(rc, entry.__name__)

    def sizes(self) -> list[int]:
        return self.nbytes[: self.count].cpu().tolist()


def make_batch(items) -> ctypes.Array:
    """items: iterable of (stream uint8 tensor, stream_bytes, out tensor, n, block)."""
    items = list(items)
    arr = (wc_batch_item * max(1, len(items)))()
    for k, (s, sb, o, n, b) in enumerate(items):
        arr[k].stream = s.data_ptr()
        arr[k].stream_bytes = sb
        arr[k].out = o.data_ptr() if n else None
        arr[k].n = n
        arr[k].block = b
        arr[k].reserved = 0
    return arr, len(items)


def decompress_batch(batch, status: torch.Tensor, stream=None):
    """Decode a batch made by ``make_batch`` in one launch per 512 tensors."""
    arr, count = batch
    rc = wc_decompress_batch(arr, count, status.data_ptr(), _stream_handle(stream))
    _check(rc, "wc_decompress_batch")


def stream_info(header: bytes):
    rc, n, block, total = wc_stream_info(header)
    _check(rc, "wc_stream_info")
    return n, block, total


def gemv(stream_bytes: torch.Tensor, rows: int, cols: int, block: int, x: torch.Tensor, *,
         nbytes: int | None = None, y: torch.Tensor | None = None,
         status: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    """y = x @ W.T with W (rows x cols BF16) given as its stream; x is (n_vec, cols)
    with n_vec in {1, 2, 4}; returns FP32 (n_vec, rows)."""
    xw = as_words(x).view(-1, cols)
    n_vec = xw.shape[0]
    if y is None:
        y = torch.empty((n_vec, rows), dtype=torch.float32, device=stream_bytes.device)
    if status is None:
        status = torch.zeros(1, dtype=torch.int32, device=stream_bytes.device)
    rc = wc_gemv(stream_bytes.data_ptr(), stream_bytes.numel() if nbytes is None else nbytes,
                 rows, cols, block, xw.data_ptr(), n_vec, y.data_ptr(), status.data_ptr(),
                 _stream_handle(stream))
    _check(rc, "wc_gemv")
    return y


def make_gemv_batch(items) -> tuple:
    """items: iterable of (stream uint8 tensor, stream_bytes, x (n_vec, cols), y (n_vec, rows), rows, cols, block)."""
    items = list(items)
    arr = (wc_gemv_item * max(1, len(items)))()
    for k, (s, sb, x, y, rows, cols, b) in enumerate(items):
        arr[k].stream = s.data_ptr()
        arr[k].stream_bytes = sb
        arr[k].x = x.data_ptr()
        arr[k].y = y.data_ptr()
        arr[k].rows, arr[k].cols, arr[k].block, arr[k].reserved = rows, cols, b, 0
    return arr, len(items)


def gemv_batch(batch, n_vec: int, status: torch.Tensor, stream=None):
    arr, count = batch
    rc = wc_gemv_batch(arr, count, n_vec, status.data_ptr(), _stream_handle(stream))
    _check(rc, "wc_gemv_batch")


GEMM_MAX_TOKENS = 128


def gemm(stream_bytes: torch.Tensor, rows: int, cols: int, block: int, x: torch.Tensor, *,
         nbytes: int | None = None, y: torch.Tensor | None = None,
         status: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    """y = x @ W.T on the tensor cores with W (rows x cols BF16) given as its stream;
    x is (tokens, cols) BF16 with 1 <= tokens <= 128; returns FP32 (tokens, rows)."""
    xw = as_words(x).view(-1, cols)
    tokens = xw.shape[0]
    if y is None:
        y = torch.empty((tokens, rows), dtype=torch.float32, device=stream_bytes.device)
    if status is None:
        status = torch.zeros(1, dtype=torch.int32, device=stream_bytes.device)
    rc = wc_gemm(stream_bytes.data_ptr(), stream_bytes.numel() if nbytes is None else nbytes,
                 rows, cols, block, xw.data_ptr(), tokens, y.data_ptr(), status.data_ptr(),
                 _stream_handle(stream))
    _check(rc, "wc_gemm")
    return y


def gemm_batch(batch, tokens: int, status: torch.Tensor, stream=None, escape: bool = False):
    """batch from make_gemv_batch (x (tokens, cols), y (tokens, rows) per item);
    escape: the streams are escape-coded (every row whole blocks)."""
    arr, count = batch
    rc = wc_gemm_batch_flags(arr, count, tokens, WC_FLAG_ESCAPE if escape else 0,
                             status.data_ptr(), _stream_handle(stream))
    _check(rc, "wc_gemm_batch_flags")


def compress_fp32(x: torch.Tensor, block: int = 1024, *, workspace: torch.Tensor | None = None,
                  stream=None) -> Compressed:
    """Compress a CUDA tensor of 32-bit words (FP32, read as bit patterns)."""
    if x.element_size() != 4:
        raise TypeError("compress_fp32 takes 32-bit words; got %s" % x.dtype)
    words = x.contiguous().view(-1).view(torch.int32)
    n = words.numel()
    cap = wc_bound_fp32(n, block)
    if cap == 0:
        raise WcodecError(WC_ERR_INVALID_ARG, "block size %r" % (block,))
    dev = words.device
    buf = torch.empty((cap + 15) // 16 * 16, dtype=torch.uint8, device=dev)
    nbytes = torch.zeros(1, dtype=torch.int64, device=dev)
    status = torch.zeros(1, dtype=torch.int32, device=dev)
    if workspace is None:
        workspace = workspace_for(n, block, dev)
    rc = wc_compress_fp32(words.data_ptr() if n else None, n, block, buf.data_ptr(), buf.numel(),
                          nbytes.data_ptr(), workspace.data_ptr(), workspace.numel(),
                          status.data_ptr(), _stream_handle(stream))
    _check(rc, "wc_compress_fp32")
    return Compressed(buf, nbytes, status, n, block, tuple(x.shape), x.dtype)


def decompress_fp32(stream_bytes: torch.Tensor, n: int, block: int, *,
                    out: torch.Tensor | None = None, status: torch.Tensor | None = None,
                    nbytes: int | None = None, stream=None) -> torch.Tensor:
    """Decode an FP32 stream into n FP32 values (``out`` if given)."""
    if out is None:
        out = torch.empty(n, dtype=torch.float32, device=stream_bytes.device)
    words = out.view(-1)
    if words.numel() != n or not words.is_contiguous() or out.element_size() != 4:
        raise ValueError("out must be a contiguous 32-bit tensor of %d elements" % n)
    if status is None:
        status = torch.zeros(1, dtype=torch.int32, device=stream_bytes.device)
    size = stream_bytes.numel() if nbytes is None else nbytes
    rc = wc_decompress_fp32(stream_bytes.data_ptr(), size, words.data_ptr() if n else None, n,
                            block, status.data_ptr(), _stream_handle(stream))
    _check(rc, "wc_decompress_fp32")
    return out


# ---------------------------------------------------------------------------
# escape-coded streams (a window of 2^w - 1 exponents per block + exceptions)
# ---------------------------------------------------------------------------
def compress_escape(x: torch.Tensor, block: int = 1024, *, workspace: torch.Tensor | None = None,
                    stream=None) -> Compressed:
    """Compress a CUDA tensor of 16-bit words into an escape-coded stream."""
    words = as_words(x)
    n = words.numel()
    cap = wc_bound_escape(n, block)
    if cap == 0:
        raise WcodecError(WC_ERR_INVALID_ARG, "block size %r" % (block,))
    dev = words.device
    buf = torch.empty((cap + 15) // 16 * 16, dtype=torch.uint8, device=dev)
    nbytes = torch.zeros(1, dtype=torch.int64, device=dev)
    status = torch.zeros(1, dtype=torch.int32, device=dev)
    if workspace is None:
        ws = wc_workspace_size_escape(n, block)
        workspace = torch.empty((ws + 15) // 16 * 16, dtype=torch.uint8, device=dev)
    rc = wc_compress_escape(words.data_ptr() if n else None, n, block, buf.data_ptr(),
                            buf.numel(), nbytes.data_ptr(), workspace.data_ptr(),
                            workspace.numel(), status.data_ptr(), _stream_handle(stream))
    _check(rc, "wc_compress_escape")
    return Compressed(buf, nbytes, status, n, block, tuple(x.shape), x.dtype, escape=True)


def decompress_escape(stream_bytes: torch.Tensor, n: int, block: int, *,
                      out: torch.Tensor | None = None, status: torch.Tensor | None = None,
                      nbytes: int | None = None, stream=None) -> torch.Tensor:
    """Decode an escape-coded stream into n 16-bit values (``out`` if given)."""
    if out is None:
        out = torch.empty(n, dtype=torch.bfloat16, device=stream_bytes.device)
    words = out.view(-1)
    if words.numel() != n or not words.is_contiguous() or out.element_size() != 2:
        raise ValueError("out must be a contiguous 16-bit tensor of %d elements" % n)
    if status is None:
        status = torch.zeros(1, dtype=torch.int32, device=stream_bytes.device)
    size = stream_bytes.numel() if nbytes is None else nbytes
    rc = wc_decompress_escape(stream_bytes.data_ptr(), size, words.data_ptr() if n else None, n,
                              block, status.data_ptr(), _stream_handle(stream))
    _check(rc, "wc_decompress_escape")
    return out


def decompress_escape_batch(batch, status: torch.Tensor, stream=None):
    """Decode escape-coded streams (a batch from ``make_batch``), one launch per 512."""
    arr, count = batch
    rc = wc_decompress_escape_batch(arr, count, status.data_ptr(), _stream_handle(stream))
    _check(rc, "wc_decompress_escape_batch")


def decompress_host_batch(batch, status: torch.Tensor, escape: bool = False, stream=None):
    """Decode streams held in page-locked host memory (a batch from ``make_batch``
    whose stream tensors are pinned CPU tensors) straight into device outputs."""
    arr, count = batch
    rc = wc_decompress_host_batch(arr, count, WC_FLAG_ESCAPE if escape else 0,
                                  status.data_ptr(), _stream_handle(stream))
    _check(rc, "wc_decompress_host_batch")


def decompress_tans_batch(batch, status: torch.Tensor, stream=None):
    """Decode tANS-coded streams (a batch from ``make_batch``, block = the chunk
    size), one launch per 256."""
    arr, count = batch
    rc = wc_decompress_tans_batch(arr, count, status.data_ptr(), _stream_handle(stream))
    _check(rc, "wc_decompress_tans_batch")


def decompress_tans(stream_bytes: torch.Tensor, n: int, chunk: int, *,
                    out: torch.Tensor | None = None, status: torch.Tensor | None = None,
                    nbytes: int | None = None, stream=None) -> torch.Tensor:
    """Decode a tANS-coded stream into n 16-bit values (``out`` if given)."""
    if out is None:
        out = torch.empty(n, dtype=torch.bfloat16, device=stream_bytes.device)
    words = out.view(-1)
    if words.numel() != n or not words.is_contiguous() or out.element_size() != 2:
        raise ValueError("out must be a contiguous 16-bit tensor of %d elements" % n)
    if status is None:
        status = torch.zeros(1, dtype=torch.int32, device=stream_bytes.device)
    size = stream_bytes.numel() if nbytes is None else nbytes
    rc = wc_decompress_tans(stream_bytes.data_ptr(), size, words.data_ptr() if n else None, n,
                            chunk, status.data_ptr(), _stream_handle(stream))
    _check(rc, "wc_decompress_tans")
    return out
