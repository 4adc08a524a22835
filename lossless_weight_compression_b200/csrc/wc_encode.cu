// wc_encode.cu -- single-pass WCB1 encoder for sm_100a.
//
// One thread block encodes one 8192-element tile (whole blocks of B elements)
// and runs every step of the encoding of "ENEC: A Lossless AI Model
// Compression Method Enabling Fast Inference on Ascend NPUs", Abstract:
//   split      each BF16 word -> exponent byte e, sign+mantissa byte s
//              (s goes straight to the mantissa plane with 16-byte stores)
//   width      per block lo = min e, hi = max e, w = bits(hi - lo); raw
//              fallback (base 0) when w == 8, else base = lo
//   scan       exclusive prefix sum of the block sizes ceil(L/8)*w: inside
//              the tile by a warp scan, across tiles by a decoupled look-back
//              (Merrill & Garland, "Single-pass Parallel Prefix Scan with
//              Decoupled Look-back", 2016) over per-tile state words
//   remap+pack v = e - base, packed by hierarchical halving (pairs, quads,
//              octets) into w bytes per octet, staged in shared memory and
//              written with 16-byte stores
// The input is read once. Tiles take their index from an atomic ticket, so a
// tile only ever waits on tiles that started before it; every wait is bounded
// by a device-timer limit after which the tile reports WC_ERR_TIMEOUT and
// marks its state word so that later tiles stop waiting too.
#include <mutex>

#include "wc_internal.cuh"

namespace wc {
namespace {

constexpr unsigned long long kFlagAggregate = 1ull << 62;  // value = this tile's bytes
constexpr unsigned long long kFlagPrefix = 2ull << 62;     // value = bytes up to and incl. this tile
constexpr unsigned long long kFlagError = 3ull << 62;      // the tile gave up
constexpr unsigned long long kValueMask = (1ull << 62) - 1;

struct EncodeArgs {
    const uint16_t* in;
    uint8_t* out;
    uint64_t* out_bytes;
    int32_t* status;
    uint32_t* control;          // [0] ticket counter, [1] internal error flag
    unsigned long long* state;  // one look-back word per tile
    Layout L;
    uint64_t ntiles;
    uint64_t timeout_ns;
    uint32_t first_ticket;
};

__device__ __forceinline__ unsigned long long load_state(const unsigned long long* p) {
    unsigned long long v;
    asm volatile("ld.relaxed.gpu.global.u64 %0, [%1];" : "=l"(v) : "l"(p) : "memory");
    return v;
}

__device__ __forceinline__ void store_state(unsigned long long* p, unsigned long long v) {
    asm volatile("st.relaxed.gpu.global.u64 [%0], %1;" ::"l"(p), "l"(v) : "memory");
}

__device__ __forceinline__ uint32_t load_flag(const uint32_t* p) {
    uint32_t v;
    asm volatile("ld.relaxed.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    return v;
}

// Two BF16 words in one u32 -> exponent bytes at bits 0-7 / 16-23 and
// sign+mantissa bytes at bits 0-7 / 16-23 (sign to bit 7, mantissa bits 6..0).
__device__ __forceinline__ void split_pair(uint32_t x, uint32_t& e2, uint32_t& s2) {
    e2 = (x >> 7) & 0x00FF00FFu;
    s2 = ((x >> 8) & 0x00800080u) | (x & 0x007F007Fu);
}

__device__ __forceinline__ uint32_t min_byte(uint32_t a) {
    a = __vminu4(a, a >> 16);
    a = __vminu4(a, a >> 8);
    return a & 0xFFu;
}

__device__ __forceinline__ uint32_t max_byte(uint32_t a) {
    a = __vmaxu4(a, a >> 16);
    a = __vmaxu4(a, a >> 8);
    return a & 0xFFu;
}

// Hierarchical halving: four w-bit values (bytes of v) -> pairs -> one quad of 4w bits.
__device__ __forceinline__ uint32_t pack_quad(uint32_t v, uint32_t w) {
    uint32_t pairs = (v & 0x00FF00FFu) | (((v >> 8) & 0x00FF00FFu) << w);
    return (pairs & 0xFFFFu) | ((pairs >> 16) << (2 * w));
}

// ... and two quads -> the octet, element t at bits [t*w, t*w + w).
__device__ __forceinline__ uint64_t pack_octet(uint32_t v_lo, uint32_t v_hi, uint32_t w) {
    return uint64_t(pack_quad(v_lo, w)) | (uint64_t(pack_quad(v_hi, w)) << (4 * w));
}

__device__ void write_container(uint8_t* out, const Layout& L, uint64_t E, int tid) {
    if (tid < 16) {
        uint64_t v = 0;
        switch (tid) {
            case 0: v = kMagic | (uint64_t(kVersion) << 32) | (uint64_t(kHeaderBytes) << 48); break;
            case 1: v = L.block; break;  // flags (bytes 12..15) = 0
            case 2: v = L.n; break;
            case 3: v = L.nb; break;
            case 4: v = L.off_hdr; break;
            case 5: v = L.off_offs; break;
            case 6: v = L.off_man; break;
            case 7: v = L.off_exp; break;
            case 8: v = E; break;
            case 9: v = L.off_exp + E; break;
            default: v = 0; break;
        }
        reinterpret_cast<uint64_t*>(out)[tid] = v;
    }
}

// Zero the padding that follows the header, offset and mantissa sections.
__device__ void write_padding(uint8_t* out, const Layout& L, int tid) {
    const uint64_t a0 = L.off_hdr + 2 * L.nb, a1 = L.off_offs + 4 * L.nb, a2 = L.off_man + L.n;
    for (uint64_t i = a0 + tid; i < L.off_offs; i += kThreads) out[i] = 0;
    for (uint64_t i = a1 + tid; i < L.off_man; i += kThreads) out[i] = 0;
    for (uint64_t i = a2 + tid; i < L.off_exp; i += kThreads) out[i] = 0;
}

__global__ void __launch_bounds__(kThreads) encode_kernel(const EncodeArgs a) {
    __shared__ __align__(16) uint8_t s_stage[kTile + 16];
    __shared__ int s_lo[kMaxBlocksPerTile], s_hi[kMaxBlocksPerTile];
    __shared__ uint32_t s_blk[kMaxBlocksPerTile];  // base | w << 8 | tile-local byte offset << 16
    __shared__ unsigned long long s_tile, s_prefix;
    __shared__ uint32_t s_total;
    __shared__ int s_abort;

    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const Layout L = a.L;

    if (L.n == 0) {  // empty tensor: the header alone
        if (blockIdx.x == 0) {
            write_container(a.out, L, 0, tid);
            if (tid == 0) *a.out_bytes = kHeaderBytes;
        }
        return;
    }

    if (tid == 0) {
        s_tile = uint64_t(atomicAdd(&a.control[0], 1u)) + a.first_ticket;
        s_abort = load_flag(&a.control[1]) != 0;
    }
    if (tid < kMaxBlocksPerTile) {
        s_lo[tid] = 255;
        s_hi[tid] = 0;
    }
    __syncthreads();
    const uint64_t t = s_tile;
    if (t >= a.ntiles) return;
    if (s_abort) {  // an earlier tile failed: mark this one so that nobody waits on it
        if (tid == 0) {
            store_state(&a.state[t], kFlagError);
            if (t == a.ntiles - 1) *a.out_bytes = 0;
        }
        return;
    }

    const uint32_t log2B = L.log2_block, B = L.block;
    const uint64_t tile_start = t * kTile;
    const uint32_t tile_n = uint32_t(min(uint64_t(kTile), L.n - tile_start));
    const uint32_t nblk = (tile_n + B - 1) >> log2B;
    const uint32_t group = min(B / kChunk, 32u);  // chunks of one block inside a warp

    // ---- split, mantissa plane, per-block min/max --------------------------------
    uint32_t E[kChunksPerThread][4];
    uint32_t nval[kChunksPerThread];
#pragma unroll
    for (int k = 0; k < kChunksPerThread; ++k) {
        const uint32_t el = uint32_t(tid + k * kThreads) * kChunk;
        const uint32_t nv = el < tile_n ? min(uint32_t(kChunk), tile_n - el) : 0u;
        nval[k] = nv;
        const uint16_t* src = a.in + tile_start + el;
        uint32_t x[8];
        if (nv == kChunk) {
            const uint4 u = ld_stream_v4(src), v = ld_stream_v4(src + 8);
            x[0] = u.x; x[1] = u.y; x[2] = u.z; x[3] = u.w;
            x[4] = v.x; x[5] = v.y; x[6] = v.z; x[7] = v.w;
        } else {
            // ragged end of the tensor: lanes past the end repeat the first
            // element, which leaves min and max unchanged
            const uint32_t first = nv ? src[0] : 0u;
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                const uint32_t h0 = (2u * i < nv) ? src[2 * i] : first;
                const uint32_t h1 = (2u * i + 1 < nv) ? src[2 * i + 1] : first;
                x[i] = h0 | (h1 << 16);
            }
        }
        uint32_t S[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            uint32_t e_a, s_a, e_b, s_b;
            split_pair(x[2 * i], e_a, s_a);
            split_pair(x[2 * i + 1], e_b, s_b);
            E[k][i] = prmt(e_a, e_b, 0x6420u);
            S[i] = prmt(s_a, s_b, 0x6420u);
        }
        uint8_t* man = a.out + L.off_man + tile_start + el;
        if (nv == kChunk) {
            st_stream_v4(man, make_uint4(S[0], S[1], S[2], S[3]));
        } else {
            for (uint32_t i = 0; i < nv; ++i) man[i] = uint8_t(S[i >> 2] >> (8 * (i & 3)));
        }
        uint32_t lo = 255u, hi = 0u;
        if (nv) {
            lo = min_byte(__vminu4(__vminu4(E[k][0], E[k][1]), __vminu4(E[k][2], E[k][3])));
            hi = max_byte(__vmaxu4(__vmaxu4(E[k][0], E[k][1]), __vmaxu4(E[k][2], E[k][3])));
        }
        for (uint32_t off = 1; off < group; off <<= 1) {
            lo = min(lo, __shfl_xor_sync(0xFFFFFFFFu, lo, off));
            hi = max(hi, __shfl_xor_sync(0xFFFFFFFFu, hi, off));
        }
        if ((lane & (group - 1)) == 0 && nv) {
            atomicMin(&s_lo[el >> log2B], int(lo));
            atomicMax(&s_hi[el >> log2B], int(hi));
        }
    }
    __syncthreads();

    // ---- warp 0: widths, sizes, tile-local scan, look-back -----------------------
    if (warp == 0) {
        uint32_t sz[2], hdr[2];
#pragma unroll
        for (int j = 0; j < 2; ++j) {
            const uint32_t i = 2 * lane + j;
            sz[j] = 0;
            hdr[j] = 0;
            if (i < nblk) {
                const uint32_t lo = s_lo[i], hi = s_hi[i], d = hi - lo;
                const uint32_t w = d ? 32u - __clz(d) : 0u;
                const uint32_t base = (w == 8u) ? 0u : lo;
                const uint32_t len = min(B, tile_n - i * B);
                sz[j] = ((len + 7) >> 3) * w;
                hdr[j] = base | (w << 8);
            }
        }
        const uint32_t pair = sz[0] + sz[1];
        uint32_t incl = pair;
#pragma unroll
        for (int off = 1; off < 32; off <<= 1) {
            const uint32_t y = __shfl_up_sync(0xFFFFFFFFu, incl, off);
            if (lane >= off) incl += y;
        }
        const uint32_t excl = incl - pair;
        if (2 * lane < nblk) s_blk[2 * lane] = hdr[0] | (excl << 16);
        if (2 * lane + 1 < nblk) s_blk[2 * lane + 1] = hdr[1] | ((excl + sz[0]) << 16);
        const uint32_t total = __shfl_sync(0xFFFFFFFFu, incl, 31);

        unsigned long long prefix = 0;
        bool failed = false, timed_out = false;
        if (t == 0) {
            if (lane == 0) store_state(&a.state[0], kFlagPrefix | total);
        } else {
            if (lane == 0) store_state(&a.state[t], kFlagAggregate | total);
            long long top = (long long)t - 1;
            const uint64_t t0 = __shfl_sync(0xFFFFFFFFu, global_timer_ns(), 0);
            while (true) {
                const long long idx = top - lane;
                const unsigned long long s = idx >= 0 ? load_state(&a.state[idx]) : kFlagPrefix;
                const uint32_t flag = uint32_t(s >> 62);
                const unsigned not_agg = __ballot_sync(0xFFFFFFFFu, flag != 1u);
                if (not_agg == 0u) {  // 32 aggregates: add them all, look further back
                    unsigned long long v = s & kValueMask;
#pragma unroll
                    for (int off = 16; off > 0; off >>= 1) v += __shfl_xor_sync(0xFFFFFFFFu, v, off);
                    prefix += v;
                    top -= 32;
                    continue;
                }
                const int first = __ffs(not_agg) - 1;
                const uint32_t fflag = __shfl_sync(0xFFFFFFFFu, flag, first);
                if (fflag == 2u) {  // an inclusive prefix: add it and the aggregates after it
                    unsigned long long v = (lane <= first) ? (s & kValueMask) : 0ull;
#pragma unroll
                    for (int off = 16; off > 0; off >>= 1) v += __shfl_xor_sync(0xFFFFFFFFu, v, off);
                    prefix += v;
                    break;
                }
                if (fflag == 3u) {  // a predecessor gave up
                    failed = true;
                    break;
                }
                // the nearest unfinished predecessor has not published yet: wait, bounded
                const bool expired = __shfl_sync(
                    0xFFFFFFFFu, int(global_timer_ns() - t0 > a.timeout_ns), 0);
                if (expired) {
                    failed = timed_out = true;
                    break;
                }
                __nanosleep(64);
            }
            if (!failed && lane == 0) store_state(&a.state[t], kFlagPrefix | (prefix + total));
        }
        if (lane == 0) {
            s_prefix = prefix;
            s_total = total;
            s_abort = failed;
            if (failed) {
                store_state(&a.state[t], kFlagError);
                atomicExch(&a.control[1], 1u);
                if (timed_out) report(a.status, kStatusTimeout);
                if (t == a.ntiles - 1) *a.out_bytes = 0;
            }
        }
    }
    __syncthreads();
    if (s_abort) return;
    const unsigned long long prefix = s_prefix;
    const uint32_t total = s_total;

    // ---- block headers and offsets -----------------------------------------------
    if (tid < nblk) {
        const uint32_t blk = s_blk[tid];
        const uint64_t b = (tile_start >> log2B) + tid;
        reinterpret_cast<uint16_t*>(a.out + L.off_hdr)[b] = uint16_t(blk & 0xFFFFu);
        reinterpret_cast<uint32_t*>(a.out + L.off_offs)[b] = uint32_t((prefix + (blk >> 16)) >> 4);
    }

    // ---- remap and pack into the staging buffer ----------------------------------
#pragma unroll
    for (int k = 0; k < kChunksPerThread; ++k) {
        const uint32_t nv = nval[k];
        if (nv == 0) continue;
        const uint32_t el = uint32_t(tid + k * kThreads) * kChunk;
        const uint32_t blk = s_blk[el >> log2B];
        const uint32_t base = blk & 0xFFu, w = (blk >> 8) & 0xFFu;
        const uint32_t dst = (blk >> 16) + ((el & (B - 1)) >> 3) * w;
        uint32_t V[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            V[i] = E[k][i] - base * 0x01010101u;  // e >= base in every byte: no borrows
            const int valid = int(nv) - 4 * i;    // lanes past the end pack as 0
            if (valid < 4) V[i] &= valid <= 0 ? 0u : (0xFFFFFFFFu >> (32 - 8 * valid));
        }
        const uint64_t o0 = pack_octet(V[0], V[1], w);
        const uint64_t o1 = pack_octet(V[2], V[3], w);
        const uint32_t nbytes = (nv > 8 ? 2u : 1u) * w;
        for (uint32_t i = 0; i < nbytes; ++i) {
            const uint64_t o = i < w ? o0 : o1;
            const uint32_t sh = 8 * (i < w ? i : i - w);
            s_stage[dst + i] = uint8_t(o >> sh);
        }
    }
    __syncthreads();

    // ---- the tile's exponent payload: 16-byte stores (the start is 16-aligned) ----
    uint8_t* dst = a.out + L.off_exp + prefix;
    for (uint32_t i = tid; i < total / 16; i += kThreads)
        st_stream_v4(dst + 16 * i, *reinterpret_cast<const uint4*>(s_stage + 16 * i));
    const uint32_t rem = total & 15u;
    if (tid < rem) dst[total - rem + tid] = s_stage[total - rem + tid];

    // ---- the last tile knows E: container header, padding, total size -----------
    if (t == a.ntiles - 1) {
        const uint64_t E = prefix + total;
        write_container(a.out, L, E, tid);
        write_padding(a.out, L, tid);
        if (tid == 0) *a.out_bytes = L.off_exp + E;
    }
}

}  // namespace

cudaError_t launch_encode(const uint16_t* in, const Layout& L, uint8_t* out, uint64_t* out_bytes,
                          void* workspace, int32_t* status, uint64_t timeout_ns,
                          uint32_t first_ticket, cudaStream_t stream) {
    const uint64_t ntiles = num_tiles(L.n);
    cudaError_t err = cudaMemsetAsync(workspace, 0, encode_workspace_bytes(L.n), stream);
    if (err != cudaSuccess) return err;
    EncodeArgs a;
    a.in = in;
    a.out = out;
    a.out_bytes = out_bytes;
    a.status = status;
    a.control = static_cast<uint32_t*>(workspace);
    a.state = reinterpret_cast<unsigned long long*>(static_cast<uint8_t*>(workspace) + 16);
    a.L = L;
    a.ntiles = ntiles;
    a.timeout_ns = timeout_ns;
    a.first_ticket = first_ticket;
    const unsigned grid = unsigned(ntiles ? ntiles : 1);
    encode_kernel<<<grid, kThreads, 0, stream>>>(a);
    return cudaGetLastError();
}

}  // namespace wc

// ---------------------------------------------------------------------------
// Allocation-free encoder entry (wc_compress_noalloc)
// ---------------------------------------------------------------------------
// Some callers cannot allocate device memory: an engine that reserves all of
// a GPU's memory for its own pools at start-up (a cudaMalloc then fails or
// fragments the pool), or a latency-critical path that must not stall on the
// device-wide synchronisation cudaMalloc/cudaFree may imply. For them the
// encoder's only scratch -- 16 bytes of control words plus one 8-byte
// look-back word per 8192-element tile -- lives in this fixed array, which
// every GPU that loads the library holds until the process exits. Its size
// caps such calls at 2^30 elements.
namespace wc {

constexpr uint64_t kNoAllocMaxElems = 1ull << 30;
constexpr uint64_t kNoAllocScratchBytes = 16 + 8 * ((kNoAllocMaxElems + kTile - 1) / kTile);

static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

namespace {
constexpr int kMaxDevices = 64;
std::mutex g_noalloc_mutex;
void* g_noalloc_ptr[kMaxDevices];  // device address of g_noalloc_scratch, per device
}  // namespace

uint64_t noalloc_max_elems() { return kNoAllocMaxElems; }

// The array's device address on the current device. The first call on a device
// looks it up with that device current; later calls reuse it. The name
// g_noalloc_scratch in host code is only a host-side stand-in, never a device
// address, so kernels always receive the looked-up pointer.
cudaError_t noalloc_scratch(void** ptr, uint64_t* bytes) {
    int dev = -1;
    cudaError_t err = cudaGetDevice(&dev);
    if (err != cudaSuccess) return err;
    if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
    std::lock_guard<std::mutex> lock(g_noalloc_mutex);
    if (g_noalloc_ptr[dev] == nullptr) {
        void* p = nullptr;
        err = cudaGetSymbolAddress(&p, g_noalloc_scratch);
        if (err != cudaSuccess) return err;
        g_noalloc_ptr[dev] = p;
    }
    *ptr = g_noalloc_ptr[dev];
    *bytes = kNoAllocScratchBytes;
    return cudaSuccess;
}

}  // namespace wc
