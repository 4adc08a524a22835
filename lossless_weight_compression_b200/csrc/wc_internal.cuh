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

struct Layout {
    uint64_t n, nb, off_hdr, off_offs, off_man, off_exp;
    uint32_t block, log2_block;
};

__host__ __device__ inline uint64_t align128(uint64_t x) { return (x + 127u) & ~uint64_t(127); }

__host__ __device__ inline bool block_ok(uint32_t B) {
    return B >= 128u && B <= 4096u && (B & (B - 1u)) == 0u;
}

__host__ __device__ inline uint32_t log2_pow2(uint32_t B) {
    uint32_t k = 0;
    while ((1u << k) < B) ++k;
    return k;
}

__host__ __device__ inline Layout make_layout(uint64_t n, uint32_t B) {
    Layout L;
    L.n = n;
    L.block = B;
    L.log2_block = log2_pow2(B);
    L.nb = (n + B - 1) >> L.log2_block;
    L.off_hdr = kHeaderBytes;
    L.off_offs = L.off_hdr + align128(2 * L.nb);
    L.off_man = L.off_offs + align128(4 * L.nb);
    L.off_exp = L.off_man + align128(n);
    return L;
}

__host__ __device__ inline uint64_t num_tiles(uint64_t n) { return (n + kTile - 1) / kTile; }

// Worst-case stream size: every block raw, 8 bytes per (possibly partial) octet.
__host__ __device__ inline uint64_t bound_bytes(uint64_t n, uint32_t B) {
    Layout L = make_layout(n, B);
    uint64_t full = n >> L.log2_block;
    uint64_t tail = n - (full << L.log2_block);
    return L.off_exp + full * B + ((tail + 7) / 8) * 8;
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

cudaError_t launch_encode(const uint16_t* in, const Layout& L, uint8_t* out, uint64_t* out_bytes,
                          void* workspace, int32_t* status, uint64_t timeout_ns,
                          uint32_t first_ticket, cudaStream_t stream);

// Bytes of workspace the encoder needs: a 16-byte control word (ticket,
// internal error flag) and one 8-byte look-back state per tile.
inline uint64_t encode_workspace_bytes(uint64_t n) { return 16 + 8 * num_tiles(n); }

cudaError_t launch_decode(const DecodeItem* items, uint32_t count, int32_t* status,
                          cudaStream_t stream);

// The allocation-free encoder's fixed scratch array (wc_encode.cu).
uint64_t noalloc_max_elems();
cudaError_t noalloc_scratch(void** ptr, uint64_t* bytes);

}  // namespace wc
