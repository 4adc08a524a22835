// wc_encode_escape.cu -- encoder of escape-coded WCB1 streams (header flags
// bit 1) for sm_100a, for one tensor or a batch of tensors.
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
// Five launches per batch of up to kEscBatchMax tensors, none of which waits
// on another thread block; the tensors' blocks (and scan chunks) are numbered
// across the batch, a scan chunk finds its tensor by binary search over the
// launch parameters and a warp walking blocks by scanning forward from its
// previous block's tensor:
//   params     one warp per block: split (the sign+mantissa bytes go straight
//              to the mantissa plane), a 256-bin exponent histogram in
//              lane-private byte counters in shared memory (incremented by
//              shared-memory reductions on the lane's word, summed with dp4a),
//              its prefix counts, and the least-cost (w, base) with all widths
//              searched at once (four lanes per width, one warp minimum);
//              writes the block header and the padded size in 16-byte units
//   reduce     one thread block per 4096 blocks of a tensor: their sizes' sum
//   top        one warp per tensor: the exclusive prefix of its chunk sums, the
//              exponent-plane size E, the container header and section padding,
//              and the stream's total size
//   down       one thread block per 4096 blocks of a tensor: the block offsets
//   pack       one warp per block, code specialised on its width: codes four at a
//              time with byte-wise arithmetic, a warp prefix count of escapes, the
//              packed codes, the exception list and zero padding built in shared
//              memory and written out with 16-byte stores
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
constexpr int kPackStageBytes = 4096;                            // a raw block's payload, B <= 4096
// params kernel: per warp 8 KB of byte counters and the 257 prefix counts
constexpr int kParamsSmem = kEscWarps * (256 * 32 + kHistWords * 4);

struct EscItem {
    const uint16_t* in;
    uint8_t* out;
    uint64_t* out_bytes;
    uint64_t n;
    uint32_t block, pad;
};

template <int MAXI>
struct EscBatch {
    uint32_t* size16;        // per block of the batch: padded payload size in 16-byte units
    uint64_t* chunk_sum;     // per chunk (4096 blocks of one tensor): their summed size16
    uint64_t* chunk_prefix;  // exclusive prefix of chunk_sum within its tensor
    uint64_t total_blocks, total_chunks;
    uint32_t count, pad;
    uint64_t block_begin[MAXI + 1];  // first block of each tensor; [count] = total
    uint64_t chunk_begin[MAXI + 1];  // first chunk of each tensor; [count] = total
    EscItem item[MAXI];
};

// The tensor that owns global unit u, given each tensor's first unit.
template <int MAXI>
__device__ __forceinline__ uint32_t owner(const uint64_t* begin, uint32_t count, uint64_t u) {
    if (MAXI == 1) return 0;
    int lo = 0, hi = int(count) - 1;
    while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (begin[mid] <= u) lo = mid; else hi = mid - 1;
    }
    return uint32_t(lo);
}

// The same, for a walk over increasing units: a scan forward from the tensor
// of the previous unit (usually one cached comparison) instead of a binary
// search of dependent loads from the launch parameters.
template <int MAXI>
__device__ __forceinline__ uint32_t owner_from(const uint64_t* begin, uint32_t count, uint64_t u,
                                               uint32_t from) {
    if constexpr (MAXI == 1) {
        return 0;
    } else {
        while (from + 1 < count && begin[from + 1] <= u) ++from;
        return from;
    }
}

__device__ __forceinline__ uint32_t block_len(const Layout& L, uint64_t b) {
    const uint64_t first = b << L.log2_block;
    return uint32_t(min(uint64_t(L.block), L.n - first));
}

// ---------------------------------------------------------------------------
// params: one warp per block
// ---------------------------------------------------------------------------
// Smallest and largest exponent of the 16-bit words in v (the exponent is the
// top byte of a word's 15-bit magnitude, so 16-bit lane minima and maxima of
// the sign-cleared words give them).
// Running per-lane minimum and maximum of the sign-cleared words, two 16-bit
// lanes at a time (mn starts at 0xFFFFFFFF, mx at 0); exponent_bounds turns
// them into exponent bytes once per block.
__device__ __forceinline__ void magnitude_range(uint4 v, uint32_t& mn, uint32_t& mx) {
    const uint32_t a = v.x & 0x7FFF7FFFu, b = v.y & 0x7FFF7FFFu, c = v.z & 0x7FFF7FFFu,
                   d = v.w & 0x7FFF7FFFu;
    asm("min.u16x2 %0, %0, %1;" : "+r"(mn) : "r"(a));
    asm("min.u16x2 %0, %0, %1;" : "+r"(mn) : "r"(b));
    asm("min.u16x2 %0, %0, %1;" : "+r"(mn) : "r"(c));
    asm("min.u16x2 %0, %0, %1;" : "+r"(mn) : "r"(d));
    asm("max.u16x2 %0, %0, %1;" : "+r"(mx) : "r"(a));
    asm("max.u16x2 %0, %0, %1;" : "+r"(mx) : "r"(b));
    asm("max.u16x2 %0, %0, %1;" : "+r"(mx) : "r"(c));
    asm("max.u16x2 %0, %0, %1;" : "+r"(mx) : "r"(d));
}

// Folds a magnitude range into an exponent range [lo, hi] (a lane that saw no
// word keeps lo = 511, above every exponent, and hi = 0).
__device__ __forceinline__ void exponent_bounds(uint32_t mn, uint32_t mx, uint32_t& lo,
                                                uint32_t& hi) {
    lo = min(lo, min(mn & 0xFFFFu, mn >> 16) >> 7);
    hi = max(hi, max(mx & 0xFFFFu, mx >> 16) >> 7);
}

template <int MAXI>
__global__ void __launch_bounds__(kEscThreads) esc_params_kernel(const __grid_constant__ EscBatch<MAXI> P) {
    // Each lane counts its own elements in byte counters laid out [exponent][lane];
    // a block gives a lane at most B / 32 <= 128 elements, so a byte never carries
    // into its neighbour. An increment is a shared-memory reduction on the
    // 32-bit word holding the lane's byte (no value returned): unlike a byte
    // read-modify-write, increments of one lane that may hit the same counter do
    // not wait for one another. Only the rows of exponents lo..hi of the block
    // are cleared, counted and summed.
    extern __shared__ __align__(16) uint8_t params_smem[];  // kParamsSmem bytes
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    uint8_t* cnt = params_smem + warp * (256 * 32);
    // the word of row e holding this lane's counter, and the lane's byte in it
    uint32_t* cnt_lane = reinterpret_cast<uint32_t*>(cnt + (lane & ~3));
    const uint32_t one = 1u << (8 * (lane & 3));
    auto count = [&](uint32_t e) { atomicAdd(cnt_lane + 8 * e, one); };
    uint32_t* h = reinterpret_cast<uint32_t*>(params_smem + kEscWarps * (256 * 32)) + warp * kHistWords;
    uint32_t it = 0;
    for (uint64_t gb = uint64_t(blockIdx.x) * kEscWarps + warp; gb < P.total_blocks;
         gb += uint64_t(gridDim.x) * kEscWarps) {
        it = owner_from<MAXI>(P.block_begin, P.count, gb, it);
        const EscItem& I = P.item[it];
        const Layout L = make_layout_escape(I.n, I.block);
        const uint64_t b = gb - P.block_begin[it];
        const uint64_t first = b << L.log2_block;
        const uint32_t len = block_len(L, b);
        const uint16_t* x = I.in + first;
        uint8_t* man = I.out + L.off_man + first;
        const uint32_t groups = len >> 3;  // whole groups of 8 elements (16 bytes)

        // pass 1: sign+mantissa bytes out, exponent range. A lane's share of a
        // block of up to 1024 elements (four 16-byte groups) is loaded at once and
        // its exponent bytes kept for pass 2; longer blocks are read again.
        constexpr uint32_t kKeep = 4;
        uint4 in[kKeep];
#pragma unroll
        for (uint32_t k = 0; k < kKeep; ++k) {
            const uint32_t g = uint32_t(lane) + 32u * k;
            in[k] = g < groups ? ld_stream_v4(x + 8 * g) : make_uint4(0u, 0u, 0u, 0u);
        }
        uint32_t mn = 0xFFFFFFFFu, mx = 0u;  // magnitude range, two lanes at a time
        uint2 keep[kKeep];  // exponent bytes of the kept groups
#pragma unroll
        for (uint32_t k = 0; k < kKeep; ++k) {
            const uint32_t g = uint32_t(lane) + 32u * k;
            if (g < groups) {
                const uint4 v = in[k];
                uint32_t s0, s1;
                split_quad(v.x, v.y, s0, keep[k].x);
                split_quad(v.z, v.w, s1, keep[k].y);
                *reinterpret_cast<uint2*>(man + 8 * g) = make_uint2(s0, s1);
                magnitude_range(v, mn, mx);
            }
        }
        for (uint32_t g = uint32_t(lane) + 32u * kKeep; g < groups; g += 32) {
            const uint4 v = ld_stream_v4(x + 8 * g);
            uint32_t s0, s1, e0, e1;
            split_quad(v.x, v.y, s0, e0);
            split_quad(v.z, v.w, s1, e1);
            *reinterpret_cast<uint2*>(man + 8 * g) = make_uint2(s0, s1);
            magnitude_range(v, mn, mx);
        }
        uint32_t lo = 511u, hi = 0u;
        exponent_bounds(mn, mx, lo, hi);
        for (uint32_t i = 8 * groups + lane; i < len; i += 32) {  // the ragged end of a tensor
            const uint32_t w16 = x[i];
            const uint32_t e = (w16 >> 7) & 0xFFu;
            man[i] = uint8_t(((w16 >> 8) & 0x80u) | (w16 & 0x7Fu));
            lo = min(lo, e);
            hi = max(hi, e);
        }
        lo = __reduce_min_sync(0xFFFFFFFFu, lo);
        hi = __reduce_max_sync(0xFFFFFFFFu, hi);
        const uint32_t span = hi - lo + 1u;  // rows in use

        // pass 2: count (the block is read again, from the caches)
        for (uint32_t r = 2 * uint32_t(lane); r < 2 * span; r += 64)  // rows lo..hi: 2 x 16 bytes each
            reinterpret_cast<uint4*>(cnt + lo * 32)[r] = make_uint4(0u, 0u, 0u, 0u),
            reinterpret_cast<uint4*>(cnt + lo * 32)[r + 1] = make_uint4(0u, 0u, 0u, 0u);
        __syncwarp();
#pragma unroll
        for (uint32_t k = 0; k < kKeep; ++k) {
            if (uint32_t(lane) + 32u * k < groups) {
#pragma unroll
                for (int t = 0; t < 8; ++t)
                    count(((t < 4 ? keep[k].x : keep[k].y) >> (8 * (t & 3))) & 0xFFu);
            }
        }
        for (uint32_t g = uint32_t(lane) + 32u * kKeep; g < groups; g += 32) {
            const uint4 v = ld_stream_v4(x + 8 * g);
            uint32_t s0, s1, e0, e1;
            split_quad(v.x, v.y, s0, e0);
            split_quad(v.z, v.w, s1, e1);
#pragma unroll
            for (int t = 0; t < 8; ++t) count(((t < 4 ? e0 : e1) >> (8 * (t & 3))) & 0xFFu);
        }
        for (uint32_t i = 8 * groups + lane; i < len; i += 32) count((uint32_t(x[i]) >> 7) & 0xFFu);
        __syncwarp();

        // h[j] <- elements with an exponent below lo + j, for j = 0..span (lane l
        // sums rows lo + l + 32k over all lanes: 32 counters = 8 words, four
        // bytes per dp4a; rows 32 bytes apart across the warp)
        uint32_t carry = 0;
        for (uint32_t r0 = 0; r0 < span; r0 += 32) {
            const uint32_t r = r0 + uint32_t(lane);
            uint32_t c = 0;
            if (r < span) {
                const uint4* row = reinterpret_cast<const uint4*>(cnt + (lo + r) * 32);
                const uint4 a = row[0], q = row[1];
                c = __dp4a(a.x, 0x01010101u, c);
                c = __dp4a(a.y, 0x01010101u, c);
                c = __dp4a(a.z, 0x01010101u, c);
                c = __dp4a(a.w, 0x01010101u, c);
                c = __dp4a(q.x, 0x01010101u, c);
                c = __dp4a(q.y, 0x01010101u, c);
                c = __dp4a(q.z, 0x01010101u, c);
                c = __dp4a(q.w, 0x01010101u, c);
            }
            uint32_t incl = c;
#pragma unroll
            for (int d = 1; d < 32; d <<= 1) {
                const uint32_t y = __shfl_up_sync(0xFFFFFFFFu, incl, d);
                if (lane >= d) incl += y;
            }
            if (r < span) h[r + 1] = carry + incl;
            carry += __shfl_sync(0xFFFFFFFFu, incl, 31);
        }
        if (lane == 0) h[0] = 0;
        __syncwarp();

        // The least-cost candidate: ties to the smaller w, then the larger base,
        // i.e. the minimum of cost << 11 | w << 8 | (255 - base) (cost <= 8 * 512 +
        // 4096 < 2^13). For a width the best base lies in [min(lo, hmax),
        // min(hi, hmax)], hmax = 255 - (2^w - 1): a window starting below lo holds
        // no more than one starting there (ties go to the larger base), one above
        // hi holds nothing. All widths are searched at once: lanes 4(w-1) ..
        // 4(w-1)+3 take width w = 1..7, every fourth base each, and one warp
        // minimum picks the winner.
        const uint32_t octets = (len + 7) >> 3;
        uint32_t best_cost = 0xFFFFFFFFu, best_w = 8, best_base = 0, best_k = 0;
        if (lo == hi) {
            best_cost = 0, best_w = 0, best_base = lo, best_k = 0;
        } else {
            uint32_t key = 0xFFFFFFFFu;
            if (lane < 28) {
                const uint32_t w = uint32_t(lane >> 2) + 1u, m = (1u << w) - 1u, hmax = 255u - m;
                const uint32_t b1 = min(hi, hmax);
                for (uint32_t base = min(lo, hmax) + uint32_t(lane & 3); base <= b1; base += 4) {
                    // elements below e: 0 up to lo, h[e - lo] inside, len above hi
                    const uint32_t top = base + m;
                    const uint32_t below_top = top > hi ? len : h[top - lo];
                    const uint32_t below_base = base <= lo ? 0u : h[base - lo];
                    const uint32_t cost = octets * w + len - (below_top - below_base);
                    key = min(key, (cost << 11) | (w << 8) | (255u - base));
                }
            }
            key = __reduce_min_sync(0xFFFFFFFFu, key);
            best_cost = key >> 11;
            best_w = (key >> 8) & 7u;
            best_base = 255u - (key & 0xFFu);
            best_k = best_cost - octets * best_w;
        }
        if (8 * octets < best_cost) best_cost = 8 * octets, best_w = 8, best_base = 0, best_k = 0;
        if (lane == 0) {
            reinterpret_cast<uint16_t*>(I.out + L.off_hdr)[b] = uint16_t(best_base | (best_w << 8));
            P.size16[gb] = (octets * best_w + best_k + 15u) >> 4;
        }
        __syncwarp();
    }
}

// ---------------------------------------------------------------------------
// the scan of the padded block sizes, per tensor
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

// The global blocks [first, end) of chunk c (all of one tensor).
template <int MAXI>
__device__ __forceinline__ void chunk_blocks(const EscBatch<MAXI>& P, uint64_t c, uint64_t& first,
                                             uint64_t& end) {
    const uint32_t it = owner<MAXI>(P.chunk_begin, P.count, c);
    first = P.block_begin[it] + (c - P.chunk_begin[it]) * kScanChunk;
    end = min(first + kScanChunk, P.block_begin[it + 1]);
}

template <int MAXI>
__global__ void __launch_bounds__(kEscThreads) esc_reduce_kernel(const __grid_constant__ EscBatch<MAXI> P) {
    __shared__ uint64_t scratch[kEscWarps];
    uint64_t cfirst, cend;
    chunk_blocks(P, blockIdx.x, cfirst, cend);
    const uint64_t first = cfirst + threadIdx.x * kScanPerThread;
    uint64_t sum = 0;
    for (uint32_t k = 0; k < kScanPerThread; ++k)
        if (first + k < cend) sum += P.size16[first + k];
    uint64_t total = 0;
    block_exclusive_scan(sum, scratch, &total);
    if (threadIdx.x == 0) P.chunk_sum[blockIdx.x] = total;
}

// One warp per tensor: the chunk prefixes, then the container header, the zero
// padding after the header, offset and mantissa sections, and the total size.
template <int MAXI>
__global__ void __launch_bounds__(kEscThreads) esc_top_kernel(const __grid_constant__ EscBatch<MAXI> P) {
    const int lane = threadIdx.x & 31;
    const uint32_t it = blockIdx.x * kEscWarps + (threadIdx.x >> 5);
    if (it >= P.count) return;
    const EscItem& I = P.item[it];
    const Layout L = make_layout_escape(I.n, I.block);
    uint64_t carry = 0;
    for (uint64_t c0 = P.chunk_begin[it]; c0 < P.chunk_begin[it + 1]; c0 += 32) {
        const uint64_t c = c0 + uint64_t(lane);
        const uint64_t v = c < P.chunk_begin[it + 1] ? P.chunk_sum[c] : 0;
        uint64_t incl = v;
#pragma unroll
        for (int d = 1; d < 32; d <<= 1) {
            const uint64_t y = __shfl_up_sync(0xFFFFFFFFu, incl, d);
            if (lane >= d) incl += y;
        }
        if (c < P.chunk_begin[it + 1]) P.chunk_prefix[c] = carry + incl - v;
        carry += __shfl_sync(0xFFFFFFFFu, incl, 31);
    }
    const uint64_t E = 16 * carry;
    uint8_t* out = I.out;
    if (lane < 16) {
        uint64_t v = 0;
        switch (lane) {
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
        reinterpret_cast<uint64_t*>(out)[lane] = v;
    }
    for (uint64_t i = L.off_hdr + 2 * L.nb + lane; i < L.off_offs; i += 32) out[i] = 0;
    for (uint64_t i = L.off_offs + 4 * L.nb + lane; i < L.off_man; i += 32) out[i] = 0;
    for (uint64_t i = L.off_man + L.n + lane; i < L.off_exp; i += 32) out[i] = 0;
    if (lane == 0) *I.out_bytes = L.off_exp + E;
}

template <int MAXI>
__global__ void __launch_bounds__(kEscThreads) esc_down_kernel(const __grid_constant__ EscBatch<MAXI> P) {
    __shared__ uint64_t scratch[kEscWarps];
    uint64_t cfirst, cend;
    chunk_blocks(P, blockIdx.x, cfirst, cend);
    const uint32_t it = owner<MAXI>(P.chunk_begin, P.count, blockIdx.x);
    const EscItem& I = P.item[it];
    const Layout L = make_layout_escape(I.n, I.block);
    const uint64_t first = cfirst + threadIdx.x * kScanPerThread;
    uint32_t v[kScanPerThread];
    uint64_t sum = 0;
#pragma unroll
    for (uint32_t k = 0; k < kScanPerThread; ++k) {
        v[k] = first + k < cend ? P.size16[first + k] : 0u;
        sum += v[k];
    }
    uint64_t total = 0;
    uint64_t run = P.chunk_prefix[blockIdx.x] + block_exclusive_scan(sum, scratch, &total);
    uint32_t* offs = reinterpret_cast<uint32_t*>(I.out + L.off_offs);
    const uint64_t local = first - P.block_begin[it];  // the tensor's own block index
#pragma unroll
    for (uint32_t k = 0; k < kScanPerThread; ++k) {
        if (first + k < cend) offs[local + k] = uint32_t(run);  // < 2^32 for n <= 2^36
        run += v[k];
    }
}

// ---------------------------------------------------------------------------
// pack: one warp per block
// ---------------------------------------------------------------------------
// Codes of four elements at width W (1..7) from their exponent bytes e4:
// r = e - base byte by byte (mod 256, no borrows between bytes); an element is
// escaped when r >= 2^W - 1, i.e. when r's top bit is set or its low seven
// bits plus 0x80 - (2^W - 1) reach 0x80. Returns the escape flags (bit 8t+7).
template <uint32_t W>
__device__ __forceinline__ uint32_t codes4(uint32_t e4, uint32_t base4, uint32_t& V) {
    constexpr uint32_t m = (1u << W) - 1u;
    const uint32_t r = ((e4 | 0x80808080u) - (base4 & 0x7F7F7F7Fu)) ^ ((e4 ^ ~base4) & 0x80808080u);
    const uint32_t t = (r & 0x7F7F7F7Fu) + (0x80u - m) * 0x01010101u;
    const uint32_t esc = (r | t) & 0x80808080u;
    const uint32_t sel = (esc >> 7) * 0xFFu;  // escaped bytes
    V = (r & ~sel) | (m * 0x01010101u & sel);
    return esc;
}

// The input words of one lane's 16-element chunk at element el of a block of
// len elements (lanes past the end: zeros).
__device__ __forceinline__ void load_chunk_words(const uint16_t* x, uint32_t el, uint32_t len,
                                                 uint32_t xw[8], uint32_t& nv) {
    nv = el < len ? min(uint32_t(kChunk), len - el) : 0u;
#pragma unroll
    for (int j = 0; j < 8; ++j) xw[j] = 0u;
    if (nv == kChunk) {
        const uint4 a = ld_stream_v4(x + el), c = ld_stream_v4(x + el + 8);
        xw[0] = a.x; xw[1] = a.y; xw[2] = a.z; xw[3] = a.w;
        xw[4] = c.x; xw[5] = c.y; xw[6] = c.z; xw[7] = c.w;
    } else {  // the ragged end of a tensor, element by element (indices fixed at compile time)
#pragma unroll
        for (uint32_t j = 0; j < 8; ++j) {
            const uint32_t lo = 2 * j < nv ? uint32_t(x[el + 2 * j]) : 0u;
            const uint32_t hi = 2 * j + 1 < nv ? uint32_t(x[el + 2 * j + 1]) : 0u;
            xw[j] = lo | (hi << 16);
        }
    }
}

// One 512-element step of a block at width W: codes, the escapes' places in the
// block's exception list (a warp prefix count on top of `carry`), the
// exceptions and the packed codes into `stage`.
template <uint32_t W>
__device__ __forceinline__ void pack_step(const uint32_t xw[8], uint32_t el,
                                          uint32_t nv, uint32_t base4, uint32_t code_bytes,
                                          uint32_t& carry, uint8_t* stage, int lane) {
    uint32_t V[4], esc[4], E[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
        uint32_t s4;
        split_quad(xw[2 * j], xw[2 * j + 1], s4, E[j]);
        if constexpr (W == 0) {
            V[j] = 0u, esc[j] = 0u;
        } else if constexpr (W == 8) {
            V[j] = E[j], esc[j] = 0u;
        } else {
            esc[j] = codes4<W>(E[j], base4, V[j]);
        }
    }
    if (nv < kChunk) {  // lanes past the end take code 0 and no escape
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const int valid = int(nv) - 4 * j;
            if (valid < 4) {
                const uint32_t keep = valid <= 0 ? 0u : (0xFFFFFFFFu >> (32 - 8 * valid));
                V[j] &= keep;
                esc[j] &= keep;
            }
        }
    }
    const uint32_t cnt = __popc(esc[0] | (esc[1] >> 1) | (esc[2] >> 2) | (esc[3] >> 3));
    uint32_t incl = cnt;
#pragma unroll
    for (int d = 1; d < 32; d <<= 1) {
        const uint32_t y = __shfl_up_sync(0xFFFFFFFFu, incl, d);
        if (lane >= d) incl += y;
    }
    uint32_t pos = code_bytes + carry + incl - cnt;
    carry += __shfl_sync(0xFFFFFFFFu, incl, 31);
    if (cnt) {
        uint32_t m16 = 0;
#pragma unroll
        for (int j = 0; j < 4; ++j) m16 |= ((esc[j] * 0x00204081u) >> 28) << (4 * j);
        // the chunk's 16 exponent bytes, already in registers
        const uint64_t e_lo = E[0] | (uint64_t(E[1]) << 32), e_hi = E[2] | (uint64_t(E[3]) << 32);
        for (; m16; m16 &= m16 - 1u) {  // exceptions in element order
            const uint32_t i = uint32_t(__ffs(int(m16))) - 1u;
            stage[pos++] = uint8_t((i < 8 ? e_lo : e_hi) >> (8 * (i & 7u)));
        }
    }
    if (nv == kChunk)
        pack_chunk<W>(V, stage + (el >> 3) * W);
    else if (nv)
        pack_chunk_tail(W, V, stage + (el >> 3) * W, (nv > 8 ? 2u : 1u) * W);
}

// Codes, exceptions and padding of one block at width W into `stage`; returns
// the block's payload bytes (a multiple of 16). Called by the whole warp; the
// loads of two steps are issued before either is processed.
template <uint32_t W>
__device__ __forceinline__ uint32_t pack_block(const uint16_t* x, uint32_t len, uint32_t base,
                                               uint8_t* stage, int lane) {
    const uint32_t code_bytes = ((len + 7) >> 3) * W;
    const uint32_t base4 = base * 0x01010101u;
    uint32_t carry = 0;  // escapes of the block before the current step
    for (uint32_t step = 0; step < len; step += 2 * 32 * kChunk) {
        const uint32_t el0 = step + uint32_t(lane) * kChunk, el1 = el0 + 32 * kChunk;
        uint32_t xa[8], xb[8], na, nb;
        load_chunk_words(x, el0, len, xa, na);
        load_chunk_words(x, el1, len, xb, nb);
        pack_step<W>(xa, el0, na, base4, code_bytes, carry, stage, lane);
        if (step + 32 * kChunk < len)  // the same for the whole warp
            pack_step<W>(xb, el1, nb, base4, code_bytes, carry, stage, lane);
    }
    const uint32_t used = code_bytes + carry, padded = (used + 15u) & ~15u;
    if (uint32_t(lane) < padded - used) stage[used + lane] = 0;
    return padded;
}

template <int MAXI>
__global__ void __launch_bounds__(kEscThreads) esc_pack_kernel(const __grid_constant__ EscBatch<MAXI> P) {
    __shared__ __align__(16) uint8_t stage_all[kEscWarps][kPackStageBytes];
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    uint8_t* stage = stage_all[warp];
    uint32_t it = 0;
    for (uint64_t gb = uint64_t(blockIdx.x) * kEscWarps + warp; gb < P.total_blocks;
         gb += uint64_t(gridDim.x) * kEscWarps) {
        it = owner_from<MAXI>(P.block_begin, P.count, gb, it);
        const EscItem& I = P.item[it];
        const Layout L = make_layout_escape(I.n, I.block);
        const uint64_t b = gb - P.block_begin[it];
        const uint32_t h = reinterpret_cast<const uint16_t*>(I.out + L.off_hdr)[b];
        const uint32_t base = h & 0xFFu, w = h >> 8;
        const uint16_t* x = I.in + (b << L.log2_block);
        const uint32_t len = block_len(L, b);
        uint8_t* payload =
            I.out + L.off_exp + 16ull * reinterpret_cast<const uint32_t*>(I.out + L.off_offs)[b];
        __syncwarp();  // the previous block's payload has left the stage
        uint32_t padded = 0;
        switch (w) {
            case 0: padded = pack_block<0>(x, len, base, stage, lane); break;
            case 1: padded = pack_block<1>(x, len, base, stage, lane); break;
            case 2: padded = pack_block<2>(x, len, base, stage, lane); break;
            case 3: padded = pack_block<3>(x, len, base, stage, lane); break;
            case 4: padded = pack_block<4>(x, len, base, stage, lane); break;
            case 5: padded = pack_block<5>(x, len, base, stage, lane); break;
            case 6: padded = pack_block<6>(x, len, base, stage, lane); break;
            case 7: padded = pack_block<7>(x, len, base, stage, lane); break;
            default: padded = pack_block<8>(x, len, base, stage, lane); break;
        }
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

// The params kernel's shared memory is above the 48 KB default: allow it once
// per device and kernel instantiation.
template <int MAXI>
cudaError_t allow_params_smem() {
    static std::mutex mu;
    static bool done[64];
    int dev = 0;
    cudaError_t err = cudaGetDevice(&dev);
    if (err != cudaSuccess) return err;
    if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
    std::lock_guard<std::mutex> lock(mu);
    if (!done[dev]) {
        err = cudaFuncSetAttribute(esc_params_kernel<MAXI>,
                                   cudaFuncAttributeMaxDynamicSharedMemorySize, kParamsSmem);
        if (err != cudaSuccess) return err;
        done[dev] = true;
    }
    return cudaSuccess;
}
uint64_t blocks_of(const EncodeItem& e) { return make_layout(e.n, e.block).nb; }

template <int MAXI>
cudaError_t encode_escape_batch(const EncodeItem* items, uint32_t count, uint8_t* ws,
                                cudaStream_t stream) {
    static_assert(sizeof(EscBatch<MAXI>) <= 32000, "launch parameters exceed the limit");
    EscBatch<MAXI> p;
    p.count = count;
    p.pad = 0;
    uint64_t blocks = 0, chunks = 0;
    for (uint32_t i = 0; i < count; ++i) {
        p.block_begin[i] = blocks;
        p.chunk_begin[i] = chunks;
        p.item[i] = EscItem{items[i].in, items[i].out, items[i].out_bytes, items[i].n,
                            items[i].block, 0u};
        blocks += blocks_of(items[i]);
        chunks += scan_chunks(blocks_of(items[i]));
    }
    p.block_begin[count] = p.total_blocks = blocks;
    p.chunk_begin[count] = p.total_chunks = chunks;
    p.size16 = reinterpret_cast<uint32_t*>(ws);
    p.chunk_sum = reinterpret_cast<uint64_t*>(ws + ((4 * blocks + 15) & ~uint64_t(15)));
    p.chunk_prefix = p.chunk_sum + chunks;
    int sms = 0;
    cudaError_t err = sm_count(&sms);
    if (err != cudaSuccess) return err;
    err = allow_params_smem<MAXI>();
    if (err != cudaSuccess) return err;
    const uint64_t warp_grid = min((blocks + kEscWarps - 1) / kEscWarps, uint64_t(8) * sms);
    if (blocks) {
        esc_params_kernel<MAXI><<<unsigned(warp_grid), kEscThreads, kParamsSmem, stream>>>(p);
        esc_reduce_kernel<MAXI><<<unsigned(chunks), kEscThreads, 0, stream>>>(p);
    }
    esc_top_kernel<MAXI><<<(count + kEscWarps - 1) / kEscWarps, kEscThreads, 0, stream>>>(p);
    if (blocks) {
        esc_down_kernel<MAXI><<<unsigned(chunks), kEscThreads, 0, stream>>>(p);
        esc_pack_kernel<MAXI><<<unsigned(warp_grid), kEscThreads, 0, stream>>>(p);
    }
    return cudaGetLastError();
}

constexpr uint32_t kEscBatchMax = 512;

}  // namespace

uint64_t escape_workspace_bytes(const EncodeItem* items, uint32_t count) {
    uint64_t total = 0;
    for (uint32_t base = 0; base < count; base += kEscBatchMax) {
        const uint32_t c = min(kEscBatchMax, count - base);
        uint64_t blocks = 0, chunks = 0;
        for (uint32_t i = 0; i < c; ++i) {
            blocks += blocks_of(items[base + i]);
            chunks += scan_chunks(blocks_of(items[base + i]));
        }
        total += ((4 * blocks + 15) & ~uint64_t(15)) + 16 * chunks + 16;
    }
    return total;
}

cudaError_t launch_encode_escape(const EncodeItem* items, uint32_t count, void* workspace,
                                 cudaStream_t stream) {
    uint8_t* ws = static_cast<uint8_t*>(workspace);
    if (count == 1) return encode_escape_batch<1>(items, 1, ws, stream);
    for (uint32_t base = 0; base < count; base += kEscBatchMax) {
        const uint32_t c = min(kEscBatchMax, count - base);
        const cudaError_t err = encode_escape_batch<kEscBatchMax>(items + base, c, ws, stream);
        if (err != cudaSuccess) return err;
        ws += escape_workspace_bytes(items + base, c);
    }
    return cudaSuccess;
}

}  // namespace wc
