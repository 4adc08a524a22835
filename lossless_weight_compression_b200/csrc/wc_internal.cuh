// wc_internal.cuh -- shared definitions of the libwcodec CUDA sources (sm_100a).
//
// The WCB1 stream layout is a function of (n, B) alone: a 128-byte container
// header, then u16 block headers, u32 block offsets, the u8 mantissa plane and
// the exponent plane, each section starting on a 128-byte boundary. Element
// split, per-block width, remap, packing and prefix sum follow "ENEC: A
// Lossless AI Model Compression Method Enabling Fast Inference on Ascend NPUs",
// Abstract; the byte layout is this library's choice.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

namespace wc {

constexpr uint32_t kMagic = 0x31424357u;  // the bytes "WCB1" as a little-endian u32
constexpr uint32_t kVersion = 1;
constexpr uint32_t kHeaderBytes = 128;
constexpr uint64_t kMaxElems = 1ull << 36;

// One thread block of either kernel works on one tile of 8192 elements: 256
// threads x 2 chunks x 16 elements. A tile always holds whole blocks
// (B <= 4096 divides 8192), so no block straddles two tiles.
constexpr int kThreads = 256;
constexpr int kChunk = 16;
constexpr int kTile = 8192;
constexpr int kChunksPerThread = kTile / (kThreads * kChunk);  // 2
constexpr int kMaxBlocksPerTile = kTile / 128;                  // 64

// Status codes written to the caller's device status word (same values as wc_status).
constexpr int32_t kStatusCorrupt = 3;
constexpr int32_t kStatusTimeout = 5;

// Header flags: bit 0 an FP32 stream, bit 1 an escape-coded stream.
constexpr uint32_t kFlagF32 = 1;
constexpr uint32_t kFlagEscape = 2;

// fp32: a stream of FP32 words, whose high halves are coded exactly as BF16
// words and whose low halves follow the mantissa plane as a raw u16 plane
// (off_low; 0 for BF16 streams). Escape-coded streams have the BF16 layout and
// flags = kFlagEscape.
struct Layout {
    uint64_t n, nb, off_hdr, off_offs, off_man, off_low, off_exp;
    uint32_t block, log2_block;
    uint32_t flags;
    bool fp32;
};

__host__ __device__ inline uint64_t align128(uint64_t x) { return (x + 127u) & ~uint64_t(127); }

__host__ __device__ inline bool block_ok(uint32_t B) {
    return B >= 128u && B <= 4096u && (B & (B - 1u)) == 0u;
}

__host__ __device__ inline uint32_t log2_pow2(uint32_t B) {
#ifdef __CUDA_ARCH__
    return uint32_t(__ffs(int(B))) - 1u;
#else
    uint32_t k = 0;
    while ((1u << k) < B) ++k;
    return k;
#endif
}

__host__ __device__ inline Layout make_layout(uint64_t n, uint32_t B, bool fp32 = false) {
    Layout L;
    L.n = n;
    L.block = B;
    L.log2_block = log2_pow2(B);
    L.nb = (n + B - 1) >> L.log2_block;
    L.off_hdr = kHeaderBytes;
    L.off_offs = L.off_hdr + align128(2 * L.nb);
    L.off_man = L.off_offs + align128(4 * L.nb);
    L.off_low = fp32 ? L.off_man + align128(n) : 0;
    L.off_exp = fp32 ? L.off_low + align128(2 * n) : L.off_man + align128(n);
    L.fp32 = fp32;
    L.flags = fp32 ? kFlagF32 : 0u;
    return L;
}

__host__ __device__ inline Layout make_layout_escape(uint64_t n, uint32_t B) {
    Layout L = make_layout(n, B, false);
    L.flags = kFlagEscape;
    return L;
}

__host__ __device__ inline uint64_t num_tiles(uint64_t n) { return (n + kTile - 1) / kTile; }

// Worst-case stream size: every block raw, 8 bytes per (possibly partial) octet.
__host__ __device__ inline uint64_t bound_bytes(uint64_t n, uint32_t B, bool fp32 = false) {
    Layout L = make_layout(n, B, fp32);
    uint64_t full = n >> L.log2_block;
    uint64_t tail = n - (full << L.log2_block);
    return L.off_exp + full * B + ((tail + 7) / 8) * 8;
}

// Worst-case escape-coded stream: every block raw, each payload padded to 16 bytes.
__host__ __device__ inline uint64_t bound_bytes_escape(uint64_t n, uint32_t B) {
    Layout L = make_layout(n, B, false);
    uint64_t full = n >> L.log2_block;
    uint64_t tail = n - (full << L.log2_block);
    return L.off_exp + full * B + (((tail + 7) / 8) * 8 + 15) / 16 * 16;
}

// ---------------------------------------------------------------------------
// PTX helpers
// ---------------------------------------------------------------------------
// Streaming 16-byte global load that is not kept in L1 (read-only data).
__device__ __forceinline__ uint4 ld_stream_v4(const void* p) {
    uint4 v;
    asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                 : "l"(p));
    return v;
}

// 16-byte global store with the evict-first hint (the output is not re-read soon).
__device__ __forceinline__ void st_stream_v4(void* p, uint4 v) {
    asm volatile("st.global.cs.v4.u32 [%0], {%1,%2,%3,%4};" ::"l"(p), "r"(v.x), "r"(v.y),
                 "r"(v.z), "r"(v.w)
                 : "memory");
}

__device__ __forceinline__ uint32_t prmt(uint32_t a, uint32_t b, uint32_t sel) {
    uint32_t r;
    asm("prmt.b32 %0, %1, %2, %3;" : "=r"(r) : "r"(a), "r"(b), "r"(sel));
    return r;
}

__device__ __forceinline__ uint64_t global_timer_ns() {
    uint64_t t;
    asm volatile("mov.u64 %0, %globaltimer;" : "=l"(t));
    return t;
}

// Record the first error in the caller's status word (NULL: not reported).
__device__ __forceinline__ void report(int32_t* status, int32_t code) {
    if (status != nullptr) atomicCAS(reinterpret_cast<int*>(status), 0, code);
}

// Every in-kernel wait on another warp or block gives up after this long.
constexpr uint64_t kWaitLimitNs = 1000000000ull;  // 1 s

// ---------------------------------------------------------------------------
// mbarrier and bulk-copy helpers (PTX)
// ---------------------------------------------------------------------------
__device__ __forceinline__ uint32_t smem_addr(const void* p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void mbar_init(unsigned long long* bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_addr(bar)), "r"(count)
                 : "memory");
}

__device__ __forceinline__ void mbar_arrive(unsigned long long* bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_addr(bar)) : "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(unsigned long long* bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_addr(bar)),
                 "r"(bytes)
                 : "memory");
}

// Test the phase with the given parity; the thread may sleep up to ~20 us in
// the instruction waiting for it (woken early when the phase completes).
__device__ __forceinline__ bool mbar_try_wait(unsigned long long* bar, uint32_t parity) {
    uint32_t done;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(done)
        : "r"(smem_addr(bar)), "r"(parity), "r"(20000u)
        : "memory");
    return done != 0;
}

// Wait for the phase of `bar` with the given parity; false if kWaitLimitNs
// passed or (abort != nullptr) another warp of the block gave up first.
// Warps off the critical path pass max_sleep_ns > 0: between polls they sleep,
// doubling from 32 ns up to that cap, and leave the issue slots to others.
__device__ __forceinline__ bool mbar_wait(unsigned long long* bar, uint32_t parity,
                                          volatile int* abort, uint32_t max_sleep_ns = 0) {
    if (mbar_try_wait(bar, parity)) return true;
    const uint64_t t0 = global_timer_ns();
    uint32_t sleep = 32;
    while (!mbar_try_wait(bar, parity)) {
        if ((abort != nullptr && *abort) || global_timer_ns() - t0 > kWaitLimitNs) return false;
        if (max_sleep_ns) {
            __nanosleep(sleep);
            sleep = min(sleep * 2u, max_sleep_ns);
        }
    }
    return true;
}

// Bulk asynchronous copy global -> this block's shared memory, completing on `bar`.
__device__ __forceinline__ void bulk_load(void* dst, const void* src, uint32_t bytes,
                                          unsigned long long* bar) {
    asm volatile(
        "cp.async.bulk.shared::cta.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
            smem_addr(dst)),
        "l"(src), "r"(bytes), "r"(smem_addr(bar))
        : "memory");
}

// Bulk asynchronous copy of this block's shared memory -> global, tracked by
// the issuing thread's bulk async-groups.
__device__ __forceinline__ void bulk_store(void* dst, const void* src, uint32_t bytes) {
    asm volatile("cp.async.bulk.global.shared::cta.bulk_group [%0], [%1], %2;" ::"l"(dst),
                 "r"(smem_addr(src)), "r"(bytes)
                 : "memory");
}

__device__ __forceinline__ void bulk_commit() {
    asm volatile("cp.async.bulk.commit_group;" ::: "memory");
}

// Wait until at most N of this thread's committed bulk groups still read shared memory.
template <int N>
__device__ __forceinline__ void bulk_wait_read() {
    asm volatile("cp.async.bulk.wait_group.read %0;" ::"n"(N) : "memory");
}

// Wait until all of this thread's committed bulk groups have completed.
__device__ __forceinline__ void bulk_wait_all() {
    asm volatile("cp.async.bulk.wait_group 0;" ::: "memory");
}

// Make this thread's generic-proxy writes to shared memory visible to bulk copies.
__device__ __forceinline__ void fence_proxy_async_smem() {
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// ---------------------------------------------------------------------------
// Launchers (defined in wc_encode.cu / wc_decode.cu)
// ---------------------------------------------------------------------------
struct DecodeItem {
    const uint8_t* stream;
    uint64_t stream_bytes;
    uint16_t* out;
    uint64_t n;
    uint32_t block;
    uint32_t reserved;
};

struct EncodeItem {
    const uint16_t* in;
    uint8_t* out;
    uint64_t* out_bytes;
    uint64_t n;
    uint32_t block;
    uint32_t reserved;
};

// Tiles of one tensor in the encoder's look-back state (an empty tensor still
// takes one, which writes its header).
__host__ __device__ inline uint64_t encode_tiles(uint64_t n) { return n ? num_tiles(n) : 1; }

// Bytes of workspace the encoder needs: a 16-byte control word (ticket,
// internal error flag) and one 8-byte look-back state per tile.
inline uint64_t encode_workspace_bytes(uint64_t tiles) { return 16 + 8 * tiles; }

// One launch for `count` tensors (the launcher splits larger batches); the
// workspace must hold encode_workspace_bytes(sum of encode_tiles) bytes.
// fp32: the inputs are FP32 words (EncodeItem::in points at n u32 words) and
// the streams are FP32 streams.
cudaError_t launch_encode(const EncodeItem* items, uint32_t count, void* workspace,
                          int32_t* status, uint64_t timeout_ns, uint32_t first_ticket,
                          cudaStream_t stream, bool fp32 = false);

// Stream kinds of the decoder: BF16 (16-bit words), FP32 (decoded into n u32
// words at DecodeItem::out) and escape-coded 16-bit streams.
enum StreamKind : int { kKindPlain = 0, kKindF32 = 1, kKindEscape = 2 };
// host_streams: every DecodeItem::stream is the device's address of page-locked
// host memory, read by the kernel over the host link (plain and escape-coded kinds).
cudaError_t launch_decode(const DecodeItem* items, uint32_t count, int32_t* status,
                          cudaStream_t stream, int kind = kKindPlain, bool host_streams = false);

// The escape-coded encoder (wc_encode_escape.cu): workspace bytes for a batch
// of tensors, and the launches that code them (five per batch of up to 512
// tensors, no cross-block waits: a per-block pass, a three-step scan of the
// block sizes, and a packing pass).
uint64_t escape_workspace_bytes(const EncodeItem* items, uint32_t count);
cudaError_t launch_encode_escape(const EncodeItem* items, uint32_t count, void* workspace,
                                 cudaStream_t stream);

struct GemvItem {
    const uint8_t* stream;  // WCB1 stream of W (rows x cols, row-major BF16)
    uint64_t stream_bytes;
    const uint16_t* x;      // n_vec x cols BF16
    float* y;               // n_vec x rows FP32
    uint32_t rows, cols, block, reserved;
};

// Fused decode + matrix-vector products for n_vec in {1, 2, 4} (wc_gemv.cu).
cudaError_t launch_gemv(const GemvItem* items, uint32_t count, uint32_t n_vec, int32_t* status,
                        cudaStream_t stream);

// Fused decode + matrix products on the tensor cores for 1..kMaxGemmTokens
// activation rows (wc_gemm.cu); one launch per kGemmBatchMax matrices.
constexpr uint32_t kMaxGemmTokens = 128;
constexpr uint32_t kGemmBatchMax = 64;
// escape: the streams are escape-coded (then every row is whole blocks).
cudaError_t launch_gemm(const GemvItem* items, uint32_t count, uint32_t tokens, bool escape,
                        int32_t* status, cudaStream_t stream);

// tANS-coded streams (wc_tans.cu): chunk sizes 1024..8192, the bytes of the
// fixed sections (header, counts, chunk offsets, mantissa plane), and the
// decoder (one launch per 256 tensors; DecodeItem::block is the chunk size).
bool tans_chunk_ok(uint32_t C);
uint64_t tans_fixed_bytes(uint64_t n, uint32_t C);
cudaError_t launch_decode_tans(const DecodeItem* items, uint32_t count, int32_t* status,
                               cudaStream_t stream);
// The encoder: the largest stream of n elements (chunk C, table log R), the
// workspace of a batch (2 KB per tensor + 4 bytes per chunk, per 256 tensors),
// and five launches per 256 tensors (EncodeItem::block is the chunk size,
// logs[i] the table log of tensor i).
uint64_t tans_bound_bytes(uint64_t n, uint32_t C, uint32_t R);
uint64_t tans_workspace_bytes(const EncodeItem* items, uint32_t count);
cudaError_t launch_encode_tans(const EncodeItem* items, const uint32_t* logs, uint32_t count,
                               void* workspace, cudaStream_t stream);

// The allocation-free encoder's fixed scratch array (wc_encode.cu).
uint64_t noalloc_max_elems();
cudaError_t noalloc_scratch(void** ptr, uint64_t* bytes);

}  // namespace wc
