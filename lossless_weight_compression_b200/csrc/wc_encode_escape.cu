// wc_encode_escape.cu -- encoder of escape-coded WCB1 streams (header flags
// bit 1) for sm_100a.
//
// A block's w-bit codes cover a window of 2^w - 1 exponents [base, base +
// 2^w - 2]; the code 2^w - 1 is an escape and the escaped elements' exponent
// bytes follow the block's codes as its exception list. (w, base) is the
// candidate of least size ceil(L/8)*w + (exceptions), ties to the smaller w,
// then to the larger base; a block of one exponent takes w = 0 and a block
// that no window shrinks is stored raw (w = 8). Codes are packed by
// hierarchical halving and blocks are placed by an exclusive prefix sum of
// their 16-byte padded sizes ("ENEC: A Lossless AI Model Compression Method
// Enabling Fast Inference on Ascend NPUs", Abstract, for the ingredients;
// "ZipServ: Fast and Memory-Efficient LLM Inference with Hardware-Aware
// Lossless Compression", Abstract, for the direction: a fixed-length format
// that decodes in constant time and shrinks weights further).
//
// Five launches, none of which waits on another thread block:
//   params     one warp per block: split (the sign+mantissa bytes go straight
//              to the mantissa plane), a 256-bin exponent histogram in shared
//              memory, its prefix counts, and for each w the window of most
//              elements (one warp maximum over all bases); writes the block
//              header and the padded size in 16-byte units
//   reduce     one thread block per 4096 sizes: their sum
//   top        one thread block: the exclusive prefix of those sums, the
//              exponent-plane size E, the container header and the section
//              padding, and the stream's total size
//   down       one thread block per 4096 sizes: the block offsets
//   pack       one warp per block: re-reads the block, codes it, packs the
//              codes, ranks the escapes with a warp prefix count, writes the
//              exception list and the payload's zero padding
// The input is read twice (params and pack); the roofline counts only the
// algorithmic bytes, 2n in and the stream out.
#include <mutex>

#include "wc_pack_core.cuh"

namespace wc {
namespace {

constexpr int kEscThreads = 256;
constexpr int kEscWarps = kEscThreads / 32;
constexpr uint32_t kScanPerThread = 16;
constexpr uint32_t kScanChunk = kScanPerThread * kEscThreads;  // 4096 block sizes per thread block
constexpr int kHistWords = 264;                                  // 256 bins + the total, padded

struct EscParams {
    const uint16_t* in;
    uint8_t* out;
    uint64_t* out_bytes;
    uint32_t* size16;        // per block: padded payload size in 16-byte units
    uint64_t* chunk_sum;     // per 4096 blocks: their summed size16
    uint64_t* chunk_prefix;  // exclusive prefix of chunk_sum
    Layout L;
    uint64_t nchunks;
};

__device__ __forceinline__ uint64_t block_len(const Layout& L, uint64_t b) {
    const uint64_t first = b << L.log2_block;
    return min(uint64_t(L.block), L.n - first);
}

// ---------------------------------------------------------------------------
// params: one warp per block
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(kEscThreads) esc_params_kernel(const EscParams P) {
    __shared__ uint32_t hist_all[kEscWarps][kHistWords];
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    uint32_t* h = hist_all[warp];
    const Layout& L = P.L;
    for (uint64_t b = uint64_t(blockIdx.x) * kEscWarps + warp; b < L.nb;
         b += uint64_t(gridDim.x) * kEscWarps) {
        for (int k = lane; k < kHistWords; k += 32) h[k] = 0;
        __syncwarp();
        const uint64_t first = b << L.log2_block;
        const uint32_t len = uint32_t(block_len(L, b));
        const uint16_t* x = P.in + first;
        uint8_t* man = P.out + L.off_man + first;
        uint32_t lo = 255u, hi = 0u;
        const uint32_t groups = len >> 3;  // whole groups of 8 elements (16 bytes)
        for (uint32_t g = lane; g < groups; g += 32) {
            const uint4 v = ld_stream_v4(x + 8 * g);
            uint32_t s0, e0, s1, e1;
            split_quad(v.x, v.y, s0, e0);
            split_quad(v.z, v.w, s1, e1);
            *reinterpret_cast<uint2*>(man + 8 * g) = make_uint2(s0, s1);
#pragma unroll
            for (int k = 0; k < 4; ++k) {
                const uint32_t ea = (e0 >> (8 * k)) & 0xFFu, eb = (e1 >> (8 * k)) & 0xFFu;
                atomicAdd(&h[ea], 1u);
                atomicAdd(&h[eb], 1u);
                lo = min(lo, min(ea, eb));
                hi = max(hi, max(ea, eb));
            }
        }
        for (uint32_t i = 8 * groups + lane; i < len; i += 32) {  // the ragged end of a tensor
            const uint32_t w16 = x[i];
            const uint32_t e = (w16 >> 7) & 0xFFu;
            man[i] = uint8_t(((w16 >> 8) & 0x80u) | (w16 & 0x7Fu));
            atomicAdd(&h[e], 1u);
            lo = min(lo, e);
            hi = max(hi, e);
        }
        __syncwarp();
        lo = __reduce_min_sync(0xFFFFFFFFu, lo);
        hi = __reduce_max_sync(0xFFFFFFFFu, hi);

        // h[e] <- number of elements with an exponent below e (h[256] = len)
        uint32_t c[8], sum = 0;
#pragma unroll
        for (int k = 0; k < 8; ++k) {
            c[k] = h[8 * lane + k];
            sum += c[k];
        }
        uint32_t incl = sum;
#pragma unroll
        for (int d = 1; d < 32; d <<= 1) {
            const uint32_t y = __shfl_up_sync(0xFFFFFFFFu, incl, d);
            if (lane >= d) incl += y;
        }
        __syncwarp();
        uint32_t run = incl - sum;
#pragma unroll
        for (int k = 0; k < 8; ++k) {
            h[8 * lane + k] = run;
            run += c[k];
        }
        if (lane == 31) h[256] = incl;
        __syncwarp();

        // the least-cost candidate: ties to the smaller w (strict comparisons in
        // increasing w), then the larger base (the maximum of count << 8 | base)
        const uint32_t octets = (len + 7) >> 3;
        uint32_t best_cost = 0xFFFFFFFFu, best_w = 8, best_base = 0, best_k = 0;
        if (lo == hi) best_cost = 0, best_w = 0, best_base = lo, best_k = 0;
#pragma unroll
        for (uint32_t w = 1; w <= 7; ++w) {
            const uint32_t m = (1u << w) - 1u;
            uint32_t key = 0;
            for (uint32_t base = lane; base + m <= 255u; base += 32)
                key = max(key, ((h[base + m] - h[base]) << 8) | base);
            key = __reduce_max_sync(0xFFFFFFFFu, key);
            const uint32_t k = len - (key >> 8);
            const uint32_t cost = octets * w + k;
            if (cost < best_cost) best_cost = cost, best_w = w, best_base = key & 0xFFu, best_k = k;
        }
        if (8 * octets < best_cost) best_cost = 8 * octets, best_w = 8, best_base = 0, best_k = 0;
        if (lane == 0) {
            reinterpret_cast<uint16_t*>(P.out + L.off_hdr)[b] = uint16_t(best_base | (best_w << 8));
            P.size16[b] = (octets * best_w + best_k + 15u) >> 4;
        }
        __syncwarp();
    }
}

// ---------------------------------------------------------------------------
// the scan of the padded block sizes
// ---------------------------------------------------------------------------
// Exclusive prefix sum of one value per thread over a 256-thread block; the
// block total goes to *total. Ends with the scratch free for reuse.
__device__ __forceinline__ uint64_t block_exclusive_scan(uint64_t v, uint64_t* scratch,
                                                         uint64_t* total) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    uint64_t incl = v;
#pragma unroll
    for (int d = 1; d < 32; d <<= 1) {
        const uint64_t y = __shfl_up_sync(0xFFFFFFFFu, incl, d);
        if (lane >= d) incl += y;
    }
    if (lane == 31) scratch[warp] = incl;
    __syncthreads();
    uint64_t warp_before = 0, all = 0;
#pragma unroll
    for (int k = 0; k < kEscWarps; ++k) {
        const uint64_t t = scratch[k];
        if (k < warp) warp_before += t;
        all += t;
    }
    __syncthreads();
    *total = all;
    return warp_before + incl - v;
}

__global__ void __launch_bounds__(kEscThreads) esc_reduce_kernel(const EscParams P) {
    __shared__ uint64_t scratch[kEscWarps];
    const uint64_t first = uint64_t(blockIdx.x) * kScanChunk + threadIdx.x * kScanPerThread;
    uint64_t sum = 0;
    for (uint32_t k = 0; k < kScanPerThread; ++k)
        if (first + k < P.L.nb) sum += P.size16[first + k];
    uint64_t total = 0;
    block_exclusive_scan(sum, scratch, &total);
    if (threadIdx.x == 0) P.chunk_sum[blockIdx.x] = total;
}

// One thread block: the chunk prefixes, then the container header, the zero
// padding after the header, offset and mantissa sections, and the total size.
__global__ void __launch_bounds__(kEscThreads) esc_top_kernel(const EscParams P) {
    __shared__ uint64_t scratch[kEscWarps];
    const Layout& L = P.L;
    uint64_t carry = 0;
    for (uint64_t base = 0; base < P.nchunks; base += kEscThreads) {
        const uint64_t c = base + threadIdx.x;
        const uint64_t v = c < P.nchunks ? P.chunk_sum[c] : 0;
        uint64_t total = 0;
        const uint64_t excl = block_exclusive_scan(v, scratch, &total);
        if (c < P.nchunks) P.chunk_prefix[c] = carry + excl;
        carry += total;
    }
    const uint64_t E = 16 * carry;
    uint8_t* out = P.out;
    if (threadIdx.x < 16) {
        uint64_t v = 0;
        switch (threadIdx.x) {
            case 0: v = kMagic | (uint64_t(kVersion) << 32) | (uint64_t(kHeaderBytes) << 48); break;
            case 1: v = L.block | (uint64_t(L.flags) << 32); break;
            case 2: v = L.n; break;
            case 3: v = L.nb; break;
            case 4: v = L.off_hdr; break;
            case 5: v = L.off_offs; break;
            case 6: v = L.off_man; break;
            case 7: v = L.off_exp; break;
            case 8: v = E; break;
            case 9: v = L.off_exp + E; break;
            default: v = 0; break;  // off_low and the reserved bytes
        }
        reinterpret_cast<uint64_t*>(out)[threadIdx.x] = v;
    }
    for (uint64_t i = L.off_hdr + 2 * L.nb + threadIdx.x; i < L.off_offs; i += kEscThreads) out[i] = 0;
    for (uint64_t i = L.off_offs + 4 * L.nb + threadIdx.x; i < L.off_man; i += kEscThreads) out[i] = 0;
    for (uint64_t i = L.off_man + L.n + threadIdx.x; i < L.off_exp; i += kEscThreads) out[i] = 0;
    if (threadIdx.x == 0) *P.out_bytes = L.off_exp + E;
}

__global__ void __launch_bounds__(kEscThreads) esc_down_kernel(const EscParams P) {
    __shared__ uint64_t scratch[kEscWarps];
    const uint64_t first = uint64_t(blockIdx.x) * kScanChunk + threadIdx.x * kScanPerThread;
    uint32_t v[kScanPerThread];
    uint64_t sum = 0;
#pragma unroll
    for (uint32_t k = 0; k < kScanPerThread; ++k) {
        v[k] = first + k < P.L.nb ? P.size16[first + k] : 0u;
        sum += v[k];
    }
    uint64_t total = 0;
    uint64_t run = P.chunk_prefix[blockIdx.x] + block_exclusive_scan(sum, scratch, &total);
    uint32_t* offs = reinterpret_cast<uint32_t*>(P.out + P.L.off_offs);
#pragma unroll
    for (uint32_t k = 0; k < kScanPerThread; ++k) {
        if (first + k < P.L.nb) offs[first + k] = uint32_t(run);  // < 2^32 for n <= 2^36
        run += v[k];
    }
}

// ---------------------------------------------------------------------------
// pack: one warp per block
// ---------------------------------------------------------------------------
// Each warp builds its block's payload (at most B <= 4096 bytes, a raw block's)
// in shared memory and writes it out with 16-byte stores.
constexpr int kPackStageBytes = 4096;

__global__ void __launch_bounds__(kEscThreads) esc_pack_kernel(const EscParams P) {
    __shared__ __align__(16) uint8_t stage_all[kEscWarps][kPackStageBytes];
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    uint8_t* stage = stage_all[warp];
    const Layout& L = P.L;
    for (uint64_t b = uint64_t(blockIdx.x) * kEscWarps + warp; b < L.nb;
         b += uint64_t(gridDim.x) * kEscWarps) {
        const uint32_t h = reinterpret_cast<const uint16_t*>(P.out + L.off_hdr)[b];
        const uint32_t base = h & 0xFFu, w = h >> 8, m = (1u << w) - 1u;
        const uint64_t first = b << L.log2_block;
        const uint32_t len = uint32_t(block_len(L, b));
        const uint32_t code_bytes = ((len + 7) >> 3) * w;
        uint8_t* payload =
            P.out + L.off_exp + 16ull * reinterpret_cast<const uint32_t*>(P.out + L.off_offs)[b];
        __syncwarp();  // the previous block's payload has left the stage
        const uint16_t* x = P.in + first;
        uint32_t carry = 0;  // escapes of the block before the current step
        for (uint32_t step = 0; step < len; step += 32 * kChunk) {
            const uint32_t el = step + uint32_t(lane) * kChunk;
            const uint32_t nv = el < len ? min(uint32_t(kChunk), len - el) : 0u;
            uint32_t xw[8] = {0u, 0u, 0u, 0u, 0u, 0u, 0u, 0u};
            if (nv == kChunk) {
                const uint4 a = ld_stream_v4(x + el), c = ld_stream_v4(x + el + 8);
                xw[0] = a.x; xw[1] = a.y; xw[2] = a.z; xw[3] = a.w;
                xw[4] = c.x; xw[5] = c.y; xw[6] = c.z; xw[7] = c.w;
            } else {
                for (uint32_t i = 0; i < nv; ++i) xw[i >> 1] |= uint32_t(x[el + i]) << (16 * (i & 1));
            }
            // codes (lanes past the end: 0) and the escape mask, element by element
            uint32_t V[4] = {0u, 0u, 0u, 0u}, m16 = 0, ex[4] = {0u, 0u, 0u, 0u};
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                uint32_t s4;
                split_quad(xw[2 * j], xw[2 * j + 1], s4, ex[j]);
#pragma unroll
                for (int t = 0; t < 4; ++t) {
                    const uint32_t i = 4u * j + t;
                    const uint32_t e = (ex[j] >> (8 * t)) & 0xFFu;
                    uint32_t code = 0;
                    if (i < nv && w != 0u) {
                        if (w == 8u) {
                            code = e;
                        } else if (e - base < m) {  // inside the window (e < base wraps)
                            code = e - base;
                        } else {
                            code = m;
                            m16 |= 1u << i;
                        }
                    }
                    V[j] |= code << (8 * t);
                }
            }
            // the chunk's first exception: a prefix count over the warp's chunks
            const uint32_t cnt = __popc(m16);
            uint32_t incl = cnt;
#pragma unroll
            for (int d = 1; d < 32; d <<= 1) {
                const uint32_t y = __shfl_up_sync(0xFFFFFFFFu, incl, d);
                if (lane >= d) incl += y;
            }
            uint32_t pos = code_bytes + carry + incl - cnt;
            carry += __shfl_sync(0xFFFFFFFFu, incl, 31);
            for (uint32_t mm = m16; mm; mm &= mm - 1u) {
                const uint32_t i = uint32_t(__ffs(int(mm))) - 1u;
                stage[pos++] = uint8_t(ex[i >> 2] >> (8 * (i & 3u)));
            }
            if (nv == kChunk)
                pack_chunk_w(w, V, stage + (el >> 3) * w);
            else if (nv)
                pack_chunk_tail(w, V, stage + (el >> 3) * w, (nv > 8 ? 2u : 1u) * w);
        }
        const uint32_t used = code_bytes + carry, padded = (used + 15u) & ~15u;
        if (uint32_t(lane) < padded - used) stage[used + lane] = 0;
        __syncwarp();
        for (uint32_t k = 16u * uint32_t(lane); k < padded; k += 16u * 32u)
            st_stream_v4(payload + k, *reinterpret_cast<const uint4*>(stage + k));
    }
}

int g_sms[64];  // SM count per device, 0 = not yet known
std::mutex g_sms_mutex;

cudaError_t sm_count(int* sms) {
    int dev = 0;
    cudaError_t err = cudaGetDevice(&dev);
    if (err != cudaSuccess) return err;
    if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
    std::lock_guard<std::mutex> lock(g_sms_mutex);
    if (g_sms[dev] == 0) {
        err = cudaDeviceGetAttribute(&g_sms[dev], cudaDevAttrMultiProcessorCount, dev);
        if (err != cudaSuccess) return err;
    }
    *sms = g_sms[dev];
    return cudaSuccess;
}

uint64_t scan_chunks(uint64_t nb) { return (nb + kScanChunk - 1) / kScanChunk; }

}  // namespace

uint64_t escape_workspace_bytes(uint64_t n, uint32_t B) {
    const Layout L = make_layout(n, B);
    return ((4 * L.nb + 15) & ~uint64_t(15)) + 16 * scan_chunks(L.nb) + 16;
}

cudaError_t launch_encode_escape(const EncodeItem& item, void* workspace, int32_t* status,
                                 cudaStream_t stream) {
    (void)status;  // nothing in these kernels waits, so nothing can time out
    EscParams p;
    p.in = item.in;
    p.out = item.out;
    p.out_bytes = item.out_bytes;
    p.L = make_layout_escape(item.n, item.block);
    p.nchunks = scan_chunks(p.L.nb);
    uint8_t* ws = static_cast<uint8_t*>(workspace);
    p.size16 = reinterpret_cast<uint32_t*>(ws);
    p.chunk_sum = reinterpret_cast<uint64_t*>(ws + ((4 * p.L.nb + 15) & ~uint64_t(15)));
    p.chunk_prefix = p.chunk_sum + p.nchunks;
    int sms = 0;
    cudaError_t err = sm_count(&sms);
    if (err != cudaSuccess) return err;
    const uint64_t warp_grid = min((p.L.nb + kEscWarps - 1) / kEscWarps, uint64_t(8) * sms);
    if (p.L.nb) {
        esc_params_kernel<<<unsigned(warp_grid), kEscThreads, 0, stream>>>(p);
        esc_reduce_kernel<<<unsigned(p.nchunks), kEscThreads, 0, stream>>>(p);
    }
    esc_top_kernel<<<1, kEscThreads, 0, stream>>>(p);
    if (p.L.nb) {
        esc_down_kernel<<<unsigned(p.nchunks), kEscThreads, 0, stream>>>(p);
        esc_pack_kernel<<<unsigned(warp_grid), kEscThreads, 0, stream>>>(p);
    }
    return cudaGetLastError();
}

}  // namespace wc
