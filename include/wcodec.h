/*
 * wcodec.h -- libwcodec: lossless compression of BF16 weight tensors with a
 * block fixed-length exponent code, on NVIDIA B200 (sm_100a).
 *
 * The method: "ENEC: A Lossless AI Model Compression Method Enabling Fast
 * Inference on Ascend NPUs", Abstract. A tensor is cut into blocks coded at one
 * fixed length each; the length is a per-block bit width (bit-width
 * quantization); values are packed two, four, then eight at a time
 * (hierarchical halving bit-packing) after a branch-free integer remap; a
 * prefix sum over block sizes places every block in the output. ZipServ
 * ("ZipServ: Fast and Memory-Efficient LLM Inference with Hardware-Aware
 * Lossless Compression", Abstract) is the reason the code is fixed-length:
 * fixed-length blocks decode in constant time per element, in parallel.
 *
 * The stream ("WCB1"), as this library fixes it (little-endian throughout;
 * sections start on 128-byte boundaries; all padding is zero):
 *   [0, 128)       container header: magic "WCB1", version 1, header size,
 *                  block size B, flags, n, nb, the four section offsets,
 *                  exponent-plane bytes E, total bytes
 *   off_hdr=128    u16 hdr[nb]   = base_b | w_b << 8
 *   off_offs       u32 offs[nb]  = start of block b's payload, in 16-byte units
 *   off_man        u8  s[n]      = sign << 7 | 7-bit mantissa of element i
 *   off_exp        E bytes       = block b at 16*offs[b]; octet j at +j*w_b;
 *                                  element t of an octet at bits [t*w, t*w+w)
 * with e = (x >> 7) & 0xFF the exponent byte, w_b = bits(max e - min e) in
 * 0..8 and base_b = min e (w_b < 8) or 0 (w_b == 8, the raw fallback).
 *
 * Conventions for every function below:
 *  - Pointers named d_* are device pointers, h_* host pointers. The caller owns
 *    every buffer. Device buffers must be 16-byte aligned.
 *  - No function allocates memory or synchronizes the device. Work is enqueued
 *    on `stream` (a cudaStream_t; 0 is the legacy default stream) and results
 *    are visible once the caller synchronizes with it.
 *  - The return value reports argument validation and launch errors only.
 *    Errors found while the kernels run (a corrupt stream, a look-back that
 *    timed out) are written to *d_status, an int32 in device memory that the
 *    caller sets to 0 beforehand; the kernels only ever write a nonzero status
 *    into it (the first error found is kept). d_status may be NULL, in which
 *    case such errors are not reported.
 *  - Block sizes B are powers of two from 128 to 4096; n <= 2^36.
 */
#ifndef WCODEC_H
#define WCODEC_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    WC_OK = 0,
    WC_ERR_INVALID_ARG = 1,      /* bad pointer, alignment, B or n */
    WC_ERR_BUFFER_TOO_SMALL = 2, /* output or workspace smaller than required */
    WC_ERR_CORRUPT_STREAM = 3,   /* stream disagrees with the WCB1 definition */
    WC_ERR_CUDA = 4,             /* a CUDA launch failed */
    WC_ERR_TIMEOUT = 5           /* a bounded in-kernel wait ran out */
} wc_status;

#define WC_HEADER_BYTES 128u
#define WC_MIN_BLOCK 128u
#define WC_MAX_BLOCK 4096u
#define WC_MAX_ELEMS (1ull << 36)

/*
 * Largest stream wc_compress can write for n elements at block size `block`:
 * every block raw, 128 + A(2nb) + A(4nb) + A(n) + sum_b 8*ceil(L_b/8) bytes,
 * A() rounding up to 128. Returns 0 if `block` or `n` is invalid.
 * (Stream layout: ENEC Abstract for the ingredients; the byte layout is this
 * library's.) Host-only, pure arithmetic.
 */
uint64_t wc_bound(uint64_t n, uint32_t block);

/*
 * Bytes of device workspace wc_compress needs for (n, block): 16 bytes of
 * control words (a tile ticket, an error flag) plus the 8-byte look-back
 * state of each 8192-element tile of the single-pass encoder (one tile for
 * n = 0). Returns 0 if `block` or `n` is invalid. Host-only.
 */
uint64_t wc_workspace_size(uint64_t n, uint32_t block);

/*
 * Compress n BF16 words (d_in, read as 16-bit patterns: NaN payloads, -0 and
 * denormals survive) into a WCB1 stream at d_out. Steps (ENEC Abstract):
 * split each word into exponent and sign+mantissa bytes; per block, the bit
 * width w = bits(max e - min e) and base; the remap e - base; hierarchical
 * halving packing of each 8 values into w bytes; an exclusive prefix sum of
 * block sizes, computed in one pass with a decoupled look-back over tiles.
 *
 *  d_in              n 16-bit words, device, 16-byte aligned
 *  d_out             out_capacity bytes, device, 16-byte aligned;
 *                    out_capacity >= wc_bound(n, block)
 *  d_out_bytes       device u64: receives the stream's total size (0 on error)
 *  d_workspace       workspace_bytes >= wc_workspace_size(n, block), device,
 *                    16-byte aligned; the call clears it on `stream` first
 *  d_status          nullable; WC_ERR_TIMEOUT if a look-back wait ran out
 * Returns WC_ERR_INVALID_ARG, WC_ERR_BUFFER_TOO_SMALL or WC_ERR_CUDA
 * without enqueuing work when the arguments are unusable. The stream is
 * byte-for-byte the same on every run and every GPU.
 */
int wc_compress(const void *d_in, uint64_t n, uint32_t block,
                void *d_out, uint64_t out_capacity, uint64_t *d_out_bytes,
                void *d_workspace, uint64_t workspace_bytes,
                int32_t *d_status, void *stream);

/*
 * One tensor of a batched compression.
 *   in, n, block: the BF16 words (device, 16-byte aligned) and the block size
 *   out, out_capacity: the stream buffer (device, 16-byte aligned),
 *                      out_capacity >= wc_bound(n, block)
 *   out_bytes: device u64 receiving the stream's size (0 on error), 8-byte aligned
 */
typedef struct {
    const void *in;
    uint64_t n;
    uint32_t block;
    uint32_t reserved; /* must be 0 */
    void *out;
    uint64_t out_capacity;
    uint64_t *out_bytes;
} wc_compress_item;

/*
 * Workspace bytes wc_compress_batch needs for these tensors (the look-back
 * state of every tile of every tensor, in parts of up to WC_BATCH_MAX
 * tensors). Returns 0 if an item has an invalid n or block. Host-only.
 */
uint64_t wc_compress_batch_workspace_size(const wc_compress_item *h_items, uint32_t count);

/*
 * Compress `count` independent tensors, each into its own WCB1 stream (every
 * stream is the one wc_compress writes for that tensor), in one launch per
 * WC_BATCH_MAX tensors. h_items is a HOST array passed to the kernel as launch
 * parameters; d_workspace (device, 16-byte aligned) holds at least
 * wc_compress_batch_workspace_size bytes and is cleared by the call on
 * `stream`. Steps as wc_compress (ENEC Abstract); tiles of all tensors share
 * one persistent grid, which removes per-tensor launch gaps for stacks of
 * many small weight tensors. Every item is checked before anything is
 * launched; errors as wc_compress.
 */
int wc_compress_batch(const wc_compress_item *h_items, uint32_t count,
                      void *d_workspace, uint64_t workspace_bytes,
                      int32_t *d_status, void *stream);

/*
 * Allocation-free variant of wc_compress. The pages have no counterpart: this
 * entry point exists for callers of the library, not for the method.
 *
 * Some callers cannot allocate device memory: an engine that reserves all of
 * a GPU's memory for its own pools at start-up (KV caches, weight arenas),
 * where a cudaMalloc fails or fragments the pool, or a latency-critical path
 * that must not stall on the device-wide synchronisation cudaMalloc and
 * cudaFree may imply. This call needs no workspace from them: the encoder's
 * look-back state lives in a fixed array inside the library,
 * WC_NOALLOC_SCRATCH_BYTES bytes of device memory that every GPU loading the
 * library holds until the process exits. Inputs, outputs and their meaning are
 * those of wc_compress.
 *  - n may not exceed WC_NOALLOC_MAX_ELEMS (2^30); a larger n returns
 *    WC_ERR_BUFFER_TOO_SMALL before anything is looked up or enqueued.
 *  - The first call on each device looks up the array's device address
 *    (cudaGetSymbolAddress) with that device current; make that first call
 *    before any stream capture. The address is kept for the life of the
 *    process: after cudaDeviceReset on a device it belongs to a context that
 *    no longer exists, so do not call this entry point on that device again
 *    in the same process.
 *  - All calls share the one array and it keeps what the last call left;
 *    every call clears the part it uses on `stream` before its kernel runs.
 *    Calls that can overlap on the GPU (unordered streams, several host
 *    threads) race on the array and can write wrong streams: serialise them.
 *  - Neither the call nor its set-up allocates memory (no cudaMalloc,
 *    cudaFree or allocating library routine).
 */
#define WC_NOALLOC_MAX_ELEMS (1ull << 30)
#define WC_NOALLOC_SCRATCH_BYTES (16ull + 8ull * (WC_NOALLOC_MAX_ELEMS / 8192ull))
int wc_compress_noalloc(const void *d_in, uint64_t n, uint32_t block,
                        void *d_out, uint64_t out_capacity,
                        uint64_t *d_out_bytes, int32_t *d_status, void *stream);

/*
 * Decompress the WCB1 stream d_stream (stream_bytes bytes, device, 16-byte
 * aligned) into n BF16 words at d_out (device, 16-byte aligned), which the
 * caller states together with `block` (wc_stream_info reads them from a host
 * copy of the header). Each element is rebuilt as
 *   x = (s & 0x80) << 8 | (base + v) << 7 | (s & 0x7F)
 * from its mantissa byte s and its w-bit value v (ZipServ Abstract: a
 * fixed-length code decodes in constant time, in parallel).
 * The kernels check the container header against (n, block), every block's
 * w <= 8 (and base 0 when w == 8), that offs is the prefix sum of the block
 * sizes and that every read stays inside stream_bytes; a failed check writes
 * WC_ERR_CORRUPT_STREAM to *d_status, and the output is then unspecified.
 * No read or write ever leaves the given buffers.
 * Returns WC_ERR_CORRUPT_STREAM at once if stream_bytes is smaller than the
 * fixed sections that (n, block) imply.
 */
int wc_decompress(const void *d_stream, uint64_t stream_bytes, void *d_out,
                  uint64_t n, uint32_t block, int32_t *d_status, void *stream);

/*
 * One tensor of a batched decode.
 *   stream, stream_bytes: the WCB1 stream (device, 16-byte aligned)
 *   out: n BF16 words (device, 16-byte aligned); block: its block size
 */
typedef struct {
    const void *stream;
    uint64_t stream_bytes;
    void *out;
    uint64_t n;
    uint32_t block;
    uint32_t reserved; /* must be 0 */
} wc_batch_item;

/*
 * Decompress `count` independent streams in as few launches as possible (one
 * launch per WC_BATCH_MAX items). h_items is a HOST array; its contents are
 * passed to the kernel as launch parameters, so the call needs no device
 * descriptor buffer and can be captured in a CUDA graph. Every check of
 * wc_decompress applies to every item; d_status collects the first error.
 */
#define WC_BATCH_MAX 512u
int wc_decompress_batch(const wc_batch_item *h_items, uint32_t count,
                        int32_t *d_status, void *stream);

/*
 * Escape-coded streams (header flags bit 1): the same fixed-length block code,
 * but a block's w-bit codes cover only a window of 2^w - 1 exponents
 * [base, base + 2^w - 2]; the code 2^w - 1 is an escape, and the escaped
 * elements' exponent bytes follow the block's codes, in element order, as its
 * exception list; each block's payload is padded to 16 bytes. Per block the
 * encoder takes the (w, base) of least size ceil(L/8)*w + exceptions (ties to
 * the smaller w, then the larger base; one exponent only: w = 0; nothing
 * smaller than raw: w = 8), with base + 2^w - 1 <= 255. On Gaussian weights
 * this settles on w = 3 with a few percent of exceptions, where the plain
 * stream needs w = 4 or 5 ("ZipServ: Fast and Memory-Efficient LLM Inference
 * with Hardware-Aware Lossless Compression", Abstract: a fixed-length format
 * that decodes in constant time and in parallel and shrinks weights further;
 * the layout is this library's). Decoding stays constant-time per element:
 * an escaped element's exception is found by a prefix count of the escapes
 * before it in its block.
 *
 *  wc_bound_escape           output capacity the encoder needs (every block
 *                            raw, payloads padded to 16 bytes); 0 if invalid
 *  wc_workspace_size_escape  device workspace bytes of wc_compress_escape
 *                            (4 bytes per block + 16 per 4096 blocks + 16)
 *  wc_compress_escape        arguments as wc_compress; d_workspace is
 *                            overwritten and need not be cleared; nothing in
 *                            it waits, so d_status is never written
 *  wc_decompress_escape      arguments as wc_decompress; the kernels check
 *                            the header (flags 2), w <= 8, base 0 when raw,
 *                            base + 2^w - 1 <= 255, that every payload holds
 *                            its codes and exceptions and has the size they
 *                            imply, and every read against stream_bytes;
 *                            WC_ERR_CORRUPT_STREAM in *d_status otherwise
 *  wc_decompress_escape_batch  wc_decompress_batch for escape-coded streams
 * A plain stream given to an escape-coded decoder, or the other way round, is
 * reported as WC_ERR_CORRUPT_STREAM.
 */
uint64_t wc_bound_escape(uint64_t n, uint32_t block);
uint64_t wc_workspace_size_escape(uint64_t n, uint32_t block);
int wc_compress_escape(const void *d_in, uint64_t n, uint32_t block, void *d_out,
                       uint64_t out_capacity, uint64_t *d_out_bytes, void *d_workspace,
                       uint64_t workspace_bytes, int32_t *d_status, void *stream);
int wc_decompress_escape(const void *d_stream, uint64_t stream_bytes, void *d_out, uint64_t n,
                         uint32_t block, int32_t *d_status, void *stream);
int wc_decompress_escape_batch(const wc_batch_item *h_items, uint32_t count,
                               int32_t *d_status, void *stream);

/*
 * wc_compress_escape over `count` tensors (h_items as for wc_compress_batch,
 * out_capacity >= wc_bound_escape(n, block) each), in five launches per 512
 * tensors; every stream equals the one wc_compress_escape writes. d_workspace
 * (device, 16-byte aligned, need not be cleared) holds at least
 * wc_compress_escape_batch_workspace_size bytes (0 if an item's n or block is
 * invalid). Every item is checked before anything is launched.
 */
uint64_t wc_compress_escape_batch_workspace_size(const wc_compress_item *h_items, uint32_t count);
int wc_compress_escape_batch(const wc_compress_item *h_items, uint32_t count, void *d_workspace,
                             uint64_t workspace_bytes, int32_t *d_status, void *stream);

/*
 * Decompression fused with the host-to-device transfer ("ENEC: A Lossless AI
 * Model Compression Method Enabling Fast Inference on Ascend NPUs", Abstract:
 * compressed weights cut the transfer in weight-transfer-bound inference).
 * The streams stay in page-locked host memory (cudaHostAlloc, cudaMallocHost
 * or cudaHostRegister; anything else returns WC_ERR_INVALID_ARG) and the
 * decoder reads each tile's bytes over the host link itself, decoding earlier
 * tiles meanwhile, into BF16 in device memory: no device buffer holds the
 * compressed streams, and only the compressed bytes cross the link.
 *   h_items / h_stream  as wc_decompress_batch / wc_decompress, except that each
 *                       stream pointer is a HOST pointer (16-byte aligned); the
 *                       host memory must not change until the work is done
 *   flags               0 for plain streams, WC_FLAG_ESCAPE for escape-coded ones
 * Checks and errors as wc_decompress (d_status); FP32 streams are not taken.
 */
#define WC_FLAG_ESCAPE 2u
int wc_decompress_host(const void *h_stream, uint64_t stream_bytes, void *d_out, uint64_t n,
                       uint32_t block, uint32_t flags, int32_t *d_status, void *stream);
int wc_decompress_host_batch(const wc_batch_item *h_items, uint32_t count, uint32_t flags,
                             int32_t *d_status, void *stream);

/*
 * FP32 tensors ("ENEC: A Lossless AI Model Compression Method Enabling Fast
 * Inference on Ascend NPUs", Abstract: the method targets AI model weights in
 * general). The high 16 bits of an FP32 word have the BF16 layout, so the
 * high halves are coded exactly as BF16 words and the low 16 bits are kept
 * raw in a plane of their own (flags bit 0 of the container header set, the
 * plane's offset at header byte 80). d_in / d_out hold n u32 words (device,
 * 16-byte aligned); everything else as wc_compress / wc_decompress, with
 * wc_bound_fp32 for the output capacity and wc_workspace_size for the
 * workspace. A decoder of one kind of stream reports the other kind as
 * WC_ERR_CORRUPT_STREAM. FP16 tensors need no entry of their own: their
 * 16-bit words go through wc_compress / wc_decompress unchanged.
 */
uint64_t wc_bound_fp32(uint64_t n, uint32_t block);
int wc_compress_fp32(const void *d_in, uint64_t n, uint32_t block, void *d_out,
                     uint64_t out_capacity, uint64_t *d_out_bytes, void *d_workspace,
                     uint64_t workspace_bytes, int32_t *d_status, void *stream);
int wc_decompress_fp32(const void *d_stream, uint64_t stream_bytes, void *d_out, uint64_t n,
                       uint32_t block, int32_t *d_status, void *stream);

/*
 * Fused decompression and matrix-vector products: for j < n_vec,
 *   y[j][r] = sum_c W[r][c] * x[j][c]
 * where W (rows x cols, row-major BF16) is given only as its WCB1 stream
 * (n = rows*cols, block size `block`): the weights are decoded on chip and
 * never written to memory ("ZipServ: Fast and Memory-Efficient LLM Inference
 * with Hardware-Aware Lossless Compression", Abstract: load compressed, compute
 * decompressed). x is n_vec x cols BF16 (device, 16-byte aligned, row-major),
 * y is n_vec x rows FP32 (device, 4-byte aligned, row-major); n_vec is 1, 2
 * or 4; cols must be a multiple of `block`. Products of two BF16 values are
 * exact in FP32 and are summed in FP32 in a fixed order, so the result is the
 * same on every run; it differs from the exact sum by at most
 * (cols-1) * 2^-24 * sum_c |W[r][c] * x[j][c]| (the standard bound of an FP32
 * sum). The stream is checked as by wc_decompress (errors to *d_status).
 */
typedef struct {
    const void *stream;
    uint64_t stream_bytes;
    const void *x;
    float *y;
    uint32_t rows, cols, block;
    uint32_t reserved; /* must be 0 */
} wc_gemv_item;

int wc_gemv(const void *d_stream, uint64_t stream_bytes, uint32_t rows, uint32_t cols,
            uint32_t block, const void *d_x, uint32_t n_vec, float *d_y,
            int32_t *d_status, void *stream);

/* wc_gemv over `count` independent matrices (one launch per 256); h_items is a
 * HOST array passed as launch parameters. */
int wc_gemv_batch(const wc_gemv_item *h_items, uint32_t count, uint32_t n_vec,
                  int32_t *d_status, void *stream);

/*
 * Fused decompression and matrix products on the tensor cores: for t < tokens,
 *   y[t][r] = sum_c W[r][c] * x[t][c]
 * with W (rows x cols, row-major BF16) given only as its WCB1 stream, as for
 * wc_gemv; the decoded weights go from the SM's own memories (shared memory,
 * then tensor memory) straight into tcgen05 tensor-core MMAs (BF16 x BF16 ->
 * FP32) and never reach device memory
 * ("ZipServ: Fast and Memory-Efficient LLM Inference with Hardware-Aware
 * Lossless Compression", Abstract: decompression fused into the GEMM). x is
 * tokens x cols BF16 (device, 16-byte aligned, row-major), y is tokens x rows
 * FP32 (device, 4-byte aligned, row-major); 1 <= tokens <= WC_GEMM_MAX_TOKENS;
 * cols must be a multiple of 128 (any valid block size). The summation order
 * is fixed, so y is the same on every run. The tensor cores' FP32 accumulation
 * is not specified to round to nearest; every output is within
 * cols * 2^-22 * sum_c |W[r][c] * x[t][c]| of the exact sum. The stream is
 * checked as by wc_decompress (errors to *d_status; an escape-coded or FP32
 * stream is reported as corrupt); a stream shorter than its planes
 * (stream_bytes below the exponent-plane offset) returns WC_ERR_CORRUPT_STREAM
 * without launching. Faster than wc_gemv at every token count, one included
 * (the token count is padded to a multiple of 16 inside); wc_gemv keeps the
 * tighter round-to-nearest bound of a plain FP32 sum.
 */
#define WC_GEMM_MAX_TOKENS 128u
int wc_gemm(const void *d_stream, uint64_t stream_bytes, uint32_t rows, uint32_t cols,
            uint32_t block, const void *d_x, uint32_t tokens, float *d_y,
            int32_t *d_status, void *stream);

/* wc_gemm over `count` independent matrices sharing one token count (one
 * launch per 64 matrices); h_items is a HOST array passed as launch
 * parameters, its x and y hold `tokens` rows each. */
int wc_gemm_batch(const wc_gemv_item *h_items, uint32_t count, uint32_t tokens,
                  int32_t *d_status, void *stream);

/*
 * wc_gemm_batch for either stream kind: flags 0 (plain WCB1 streams, exactly
 * wc_gemm_batch) or WC_FLAG_ESCAPE (escape-coded streams, as written by
 * wc_compress_escape). The escape-coded product is the combination the
 * ZipServ abstract describes ("ZipServ: Fast and Memory-Efficient LLM
 * Inference with Hardware-Aware Lossless Compression", Abstract: a compact
 * fixed-length format decoded in constant time, in parallel, directly into the
 * tensor-core operands): an element's code sits at a closed-form position and
 * an escaped element takes the next byte of its block's exception list. For
 * escape-coded streams every row must be whole blocks (cols a multiple of
 * block; else WC_ERR_INVALID_ARG). Results, bound and determinism as
 * wc_gemm. The stream is checked for what the kernel reads (each block's width
 * and window, the offset chain against the codes, the exception list against
 * the escape count and outside the window, every read inside stream_bytes);
 * a stream of the other kind is reported as corrupt. Any other flags value:
 * WC_ERR_INVALID_ARG.
 */
int wc_gemm_batch_flags(const wc_gemv_item *h_items, uint32_t count, uint32_t tokens,
                        uint32_t flags, int32_t *d_status, void *stream);

/*
 * tANS-coded streams (header flags 4): the exponent bytes entropy-coded by
 * tabled asymmetric numeral systems ("MINE: Entropy-coded Memory-efficient
 * Inference for Large Language Models", Abstract: a GPU entropy coder of the
 * tANS family, dtANS-LLM, exploiting the non-uniform distribution of weights,
 * with hyper-parameters that trade compression ratio against decoding cost;
 * the format is this library's reading). One normalized histogram per tensor
 * with 2^table_log states (table_log 8..12); the tensor is cut into chunks of
 * `chunk` elements (1024, 2048, 4096 or 8192), each coded as 32 interleaved
 * lane streams (lane l: the chunk's elements l, l + 32, ...) that share one
 * stream of 32-bit words, taken in turn by the lanes holding fewer than
 * table_log bits; the sign+mantissa bytes stay raw. Unlike the fixed-length
 * streams, a lane's position in the word stream is only known after its
 * previous element ("ZipServ ...", Abstract: variable-length codes break SIMT
 * parallelism), so one warp decodes one chunk step by step.
 * Layout: the WCB1 header (flags 4, the chunk size in the block field, the
 * table log at byte 88), 256 u16 normalized counts at byte 128, u32 chunk
 * offsets (16-byte units) at byte 640, the mantissa plane, then per chunk 32
 * u16 first states, the words and zero padding to 16 bytes.
 *
 *  wc_bound_tans        output capacity the encoder needs; 0 if invalid
 *  wc_compress_tans_batch_workspace_size
 *                       device workspace of wc_compress_tans[_batch]: 2 KB per
 *                       tensor and 4 bytes per chunk (per WC_BATCH_MAX tensors)
 *  wc_compress_tans[_batch]
 *                       encode (items' block = the chunk size): five launches
 *                       per WC_BATCH_MAX tensors, none waiting on another
 *                       thread block; the workspace is overwritten (cleared by
 *                       the call on `stream`); *out_bytes receives each size
 *  wc_decompress_tans[_batch]
 *                       decode (block = the chunk size): one launch per 256
 *                       tensors. The kernels check the header, that the counts
 *                       sum to 2^table_log, every chunk's offsets and first
 *                       states, every word read against its chunk's payload,
 *                       and that every lane ends in state 0 with fewer than 4
 *                       unused words; WC_ERR_CORRUPT_STREAM in *d_status
 *                       otherwise, with every read inside stream_bytes. A
 *                       stream shorter than its fixed sections returns
 *                       WC_ERR_CORRUPT_STREAM without launching.
 * Device pointers 16-byte aligned; the library allocates nothing.
 */
uint64_t wc_bound_tans(uint64_t n, uint32_t chunk, uint32_t table_log);
uint64_t wc_compress_tans_batch_workspace_size(const wc_compress_item *h_items, uint32_t count);
int wc_compress_tans(const void *d_in, uint64_t n, uint32_t chunk, uint32_t table_log,
                     void *d_out, uint64_t out_capacity, uint64_t *d_out_bytes,
                     void *d_workspace, uint64_t workspace_bytes, void *stream);
int wc_compress_tans_batch(const wc_compress_item *h_items, uint32_t count, uint32_t table_log,
                           void *d_workspace, uint64_t workspace_bytes, void *stream);
int wc_decompress_tans(const void *d_stream, uint64_t stream_bytes, void *d_out, uint64_t n,
                       uint32_t chunk, int32_t *d_status, void *stream);
int wc_decompress_tans_batch(const wc_batch_item *h_items, uint32_t count, int32_t *d_status,
                             void *stream);

/*
 * Parse a host copy of a stream's first `header_bytes` (>= 128) bytes. Fills
 * n, block and total_bytes (any may be NULL). Returns WC_ERR_CORRUPT_STREAM
 * if the header is not a WCB1 version-1 header consistent with itself (BF16,
 * FP32, escape-coded or tANS-coded stream; header bytes 12..15 say which; for
 * a tANS-coded stream `block` is its chunk size).
 */
int wc_stream_info(const void *h_header, uint64_t header_bytes,
                   uint64_t *n, uint32_t *block, uint64_t *total_bytes);

/* A static, human-readable name for a status code. */
const char *wc_status_string(int status);

/*
 * Test hook for the bounded waits of wc_compress. Runs the same encoder,
 * except that no thread block ever takes tile 0, so the look-back of every
 * later tile waits on a flag that nothing sets. Each such wait gives up after
 * timeout_ns nanoseconds (device global timer) and the call ends with
 * WC_ERR_TIMEOUT in *d_status, leaving the device usable. Needs n large
 * enough for at least two 8192-element tiles. Arguments as wc_compress.
 */
int wc_debug_compress_stalled(const void *d_in, uint64_t n, uint32_t block,
                              void *d_out, uint64_t out_capacity,
                              uint64_t *d_out_bytes, void *d_workspace,
                              uint64_t workspace_bytes, int32_t *d_status,
                              uint64_t timeout_ns, void *stream);

#ifdef __cplusplus
}
#endif

#endif /* WCODEC_H */
