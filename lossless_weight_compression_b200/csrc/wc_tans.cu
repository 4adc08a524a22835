// wc_tans.cu -- decoder of tANS-coded streams (header flags 4) for sm_100a.
//
// The exponent bytes of a tensor are entropy-coded by tabled asymmetric
// numeral systems with one normalized histogram per tensor (2^R states); the
// tensor is cut into chunks of C elements, each coded as 32 interleaved lane
// streams (lane l: the chunk's elements l, l + 32, ...) sharing one stream of
// 32-bit words that the lanes take in turn, step by step. The sign+mantissa
// bytes stay raw. "MINE: Entropy-coded Memory-efficient Inference for Large
// Language Models", Abstract: a GPU entropy coder of the tANS family whose
// hyper-parameters (here R and C) trade compression ratio against decoding
// cost; its variable-length codes are what "ZipServ: Fast and
// Memory-Efficient LLM Inference with Hardware-Aware Lossless Compression",
// Abstract, contrasts with fixed-length formats: each lane's position in the
// word stream is only known after the previous step.
//
// One warp decodes one chunk: lane l owns the chunk's lane stream l. Per step
// the lanes holding fewer than R bits take the next words in lane order (a
// ballot and a prefix count), then every lane decodes one exponent with one
// table lookup (state -> exponent, bits to read, next state base). A thread
// block (8 warps) works through a contiguous range of 8-chunk tiles; it builds
// the tensor's decoding table in shared memory whenever its tiles move to a
// new tensor, and each warp stages its chunk's payload and mantissa bytes with
// one bulk copy (payloads larger than C/2 + 512 bytes, which only poorly
// compressible chunks reach, are read from global memory instead). A full
// chunk runs a step loop without per-element bounds tests: word indices are
// clamped into the payload and the chunk is checked once at its end. A stream
// that breaks the format writes WC_ERR_CORRUPT_STREAM to the status word.
#include <mutex>

#include "wc_decode_core.cuh"
#include "wc_pack_core.cuh"

namespace wc {
namespace {

constexpr int kTansWarps = 8;
constexpr int kTansThreads = 32 * kTansWarps;
constexpr uint32_t kTansMaxLog = 12;
constexpr uint32_t kTansMinLog = 8;
constexpr uint32_t kTansTable = 1u << kTansMaxLog;  // entries
constexpr uint32_t kTansSlack = 512;

// Staged payload bytes per warp for chunk size C: a payload of Gaussian
// weights takes about C/3 bytes; larger ones are read from global memory.
__host__ __device__ constexpr uint32_t tans_pay_stage(uint32_t C) { return C / 2 + kTansSlack; }
// per warp: the payload stage, then the chunk's mantissa bytes
__host__ __device__ constexpr uint32_t tans_stage_bytes(uint32_t C) { return tans_pay_stage(C) + C; }
// A full chunk takes at most one word per lane every other step (a word
// leaves at least 32 - 12 bits after the step that takes it): 16 words per
// step, C/2 words in all. A lane reads word index at most C/2 (a lane that
// takes none reads the index after the pair's last), i.e. below 68 + 2C bytes
// past the start of the warp's payload stage. The allocation extends that far
// past the last warp's stage, so word reads of the staged path need no clamp:
// a corrupt chunk reads stale bytes inside the block's shared memory and fails
// its end checks.
__host__ __device__ constexpr uint32_t tans_read_slack(uint32_t C) {
    return 80u + 2u * C > tans_stage_bytes(C) ? 80u + 2u * C - tans_stage_bytes(C) : 0u;
}

template <int MAXI>
struct TansParams {
    DecodeItem item[MAXI];            // block = the chunk size C
    uint64_t tile_begin[MAXI + 1];    // first tile of each tensor; [count] = total
    int32_t* status;
    uint32_t count;
    uint32_t max_chunk;               // the largest C of the batch (staging size)
};

// C is a power of two (1024..8192): chunk counts by a shift, not a 64-bit division
// (which the decoder would otherwise run for every chunk).
__host__ __device__ inline uint32_t tans_log2(uint32_t C) {
#ifdef __CUDA_ARCH__
    return uint32_t(__ffs(int(C))) - 1u;
#else
    return uint32_t(__builtin_ctz(C));
#endif
}
__host__ __device__ inline uint64_t tans_chunks(uint64_t n, uint32_t C) {
    return (n + C - 1) >> tans_log2(C);
}
__host__ __device__ inline uint64_t tans_tiles(uint64_t n, uint32_t C) {
    return (tans_chunks(n, C) + kTansWarps - 1) / kTansWarps;
}

struct TansLayout {
    uint64_t nb, off_offs, off_man, off_exp;
};

__host__ __device__ inline TansLayout tans_layout(uint64_t n, uint32_t C) {
    TansLayout L;
    L.nb = tans_chunks(n, C);
    L.off_offs = kHeaderBytes + 512;
    L.off_man = L.off_offs + align128(4 * L.nb);
    L.off_exp = L.off_man + align128(n);
    return L;
}

__device__ __forceinline__ uint32_t lanemask_lt() {
    uint32_t m;
    asm("mov.u32 %0, %%lanemask_lt;" : "=r"(m));
    return m;
}

template <int MAXI>
__device__ __forceinline__ uint32_t tans_find_item(const TansParams<MAXI>& P, uint64_t t) {
    int lo = 0, hi = int(P.count) - 1;
    while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (P.tile_begin[mid] <= t) lo = mid; else hi = mid - 1;
    }
    return uint32_t(lo);
}

struct TansShared {
    uint32_t* table;   // kTansTable entries: bits | exponent << 7 | 4 next << 18
    uint32_t* cum;     // 257 cumulative counts
    uint32_t* seen;    // 256 running occurrence counts (table build)
    uint32_t* info;    // [0] R, [1] the tensor is usable (1) or not (0)
    unsigned long long* bar;  // one per warp
    uint8_t* stage;    // per warp: tans_stage_bytes(max chunk)
};

// The container header and the counts of item I: checks, then the decoding
// table of the normalized counts. Called by all threads of the block.
template <int MAXI>
__device__ void tans_build(const TansParams<MAXI>& P, const DecodeItem& I, TansShared& S) {
    const int tid = threadIdx.x;
    const uint8_t* st = I.stream;
    const TansLayout L = tans_layout(I.n, I.block);
    if (tid == 0) {
        bool bad = ld_u64(st) != (kMagic | (uint64_t(kVersion) << 32) | (uint64_t(kHeaderBytes) << 48));
        bad |= ld_u64(st + 8) != (uint64_t(I.block) | (uint64_t(4) << 32));
        bad |= ld_u64(st + 16) != I.n || ld_u64(st + 24) != L.nb;
        bad |= ld_u64(st + 32) != kHeaderBytes || ld_u64(st + 40) != L.off_offs;
        bad |= ld_u64(st + 48) != L.off_man || ld_u64(st + 56) != L.off_exp;
        const uint64_t E = ld_u64(st + 64), total = ld_u64(st + 72);
        bad |= total != L.off_exp + E || total > I.stream_bytes || ld_u64(st + 80) != 0;
        const uint32_t R = uint32_t(ld_u64(st + 88));
        bad |= R < kTansMinLog || R > kTansMaxLog;
        for (int k = 96; k < 128; k += 8) bad |= ld_u64(st + k) != 0;
        S.info[0] = bad ? kTansMinLog : R;
        S.info[1] = bad ? 0u : 1u;
        if (bad) report(P.status, kStatusCorrupt);
    }
    __syncthreads();
    const uint32_t R = S.info[0], Lst = 1u << R;
    // counts and their exclusive prefix sum (threads 0..255, one count each)
    const uint32_t f = tid < 256 ? uint32_t(reinterpret_cast<const uint16_t*>(st + kHeaderBytes)[tid]) : 0u;
    uint32_t incl = f;
    const int lane = tid & 31, warp = tid >> 5;
#pragma unroll
    for (int d = 1; d < 32; d <<= 1) {
        const uint32_t y = __shfl_up_sync(0xFFFFFFFFu, incl, d);
        if (lane >= d) incl += y;
    }
    if (lane == 31) S.seen[warp] = incl;  // warp totals, briefly
    // the zero padding after the chunk offsets and after the mantissa plane
    // (each under 128 bytes; inside the stream once the header is valid)
    bool pad_bad = false;
    if (S.info[1]) {
        const uint64_t o1 = L.off_offs + 4 * L.nb, o2 = L.off_man + I.n;
        if (uint64_t(tid) < L.off_man - o1) pad_bad |= st[o1 + tid] != 0;
        if (uint64_t(tid) < L.off_exp - o2) pad_bad |= st[o2 + tid] != 0;
    }
    const bool any_pad_bad = __syncthreads_or(pad_bad) != 0;
    uint32_t before = 0;
    for (int k = 0; k < warp; ++k) before += S.seen[k];
    __syncthreads();
    if (tid < 256) {
        S.cum[tid] = before + incl - f;
        S.seen[tid] = f;  // occurrence counters start at f
        if (tid == 255) {
            S.cum[256] = before + incl;
            if (before + incl != Lst || S.info[1] == 0 || any_pad_bad) {
                if (S.info[1]) report(P.status, kStatusCorrupt);
                S.info[1] = 0;
            }
        }
    }
    __syncthreads();
    if (S.info[1] == 0) return;  // every thread reads the same value
    // spread: the k-th slot (exponents in order, f[e] slots each) goes to state
    // k * step mod L; slot k belongs to the largest e with cum[e] <= k
    const uint32_t step = (Lst >> 1) + (Lst >> 3) + 3u;
    for (uint32_t k = tid; k < Lst; k += kTansThreads) {
        int lo = 0, hi = 255;
        while (lo < hi) {
            const int mid = (lo + hi + 1) >> 1;
            if (S.cum[mid] <= k) lo = mid; else hi = mid - 1;
        }
        S.table[(k * step) & (Lst - 1u)] = uint32_t(lo);
    }
    __syncthreads();
    // state X holds the v-th occurrence of its exponent (v from f[e], in
    // increasing X): bits = R - floor(log2 v), next = v * 2^bits - L. One warp
    // walks the states in order, 32 at a time.
    if (warp == 0) {
        for (uint32_t x0 = 0; x0 < Lst; x0 += 32) {
            const uint32_t X = x0 + uint32_t(lane);
            const uint32_t e = S.table[X] & 0xFFu;
            const uint32_t grp = __match_any_sync(0xFFFFFFFFu, e);
            const uint32_t v = S.seen[e] + __popc(grp & lanemask_lt());
            __syncwarp();
            if ((grp >> lane) == 1u) S.seen[e] = v + 1u;  // the group's highest lane
            const uint32_t nb = R - (31u - __clz(v));
            S.table[X] = nb | (e << 7) | ((((v << nb) - Lst) * 4u) << 18);
            __syncwarp();
        }
    }
    __syncthreads();
}

__device__ __forceinline__ uint32_t smem_addr(const void* p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}
__device__ __forceinline__ uint32_t lds_u32(uint32_t a) {
    uint32_t v;
    asm volatile("ld.shared.u32 %0, [%1];" : "=r"(v) : "r"(a));
    return v;
}
__device__ __forceinline__ uint32_t lds_u8(uint32_t a) {
    uint32_t v;
    asm volatile("ld.shared.u8 %0, [%1];" : "=r"(v) : "r"(a));
    return v;
}
// the low n bits set (n <= 32)
__device__ __forceinline__ uint32_t low_mask(uint32_t n) {
    uint32_t m;
    asm("bmsk.clamp.b32 %0, 0, %1;" : "=r"(m) : "r"(n));
    return m;
}

// One lane's decoder: the shared-memory address of its state's table entry,
// its bit buffer (hi:lo, cnt bits, nothing above them) and the number of words
// the warp has taken. At a refill cnt < R <= 12, so hi is zero then.
struct TansLane {
    uint32_t xa, lo, hi, cnt, p;
};

// A word taken while fewer than 32 bits are held (hi is zero then) goes above them.
__device__ __forceinline__ void tans_insert(TansLane& d, uint32_t w) {
    d.lo |= w << d.cnt;
    d.hi = __funnelshift_l(w, 0u, d.cnt);  // w >> (32 - cnt), 0 for cnt = 0
    d.cnt += 32u;
}

// The element of table entry t: read its bits, move to the next state, write
// the BF16 word (sign and mantissa bits from the staged byte at ma, exponent
// bits from the entry, in one select).
__device__ __forceinline__ void tans_decode(TansLane& d, uint32_t t, uint32_t tbase, uint32_t ma,
                                            uint16_t* o) {
    const uint32_t nb = t & 15u;
    d.xa = tbase + (t >> 18) + ((d.lo & low_mask(nb)) << 2);
    d.lo = __funnelshift_r(d.lo, d.hi, nb);
    d.hi >>= nb;
    d.cnt -= nb;
    const uint32_t x = lds_u8(ma) * 0x101u;  // the byte twice: sign at bit 15
    *o = uint16_t((x & 0x807Fu) | (t & 0x7F80u));
}

// One step of lane `lane` for element i: refill (words in lane order among the
// lanes holding fewer than R bits; the index is clamped into the payload, so a
// corrupt stream reads stale words and is caught by the word count at the end),
// then one table lookup: exponent, bits to read, next state. A table entry is
// nb | e << 7 | 4 next << 18; the output takes the sign and mantissa bits of s
// and the exponent bits of the entry in one select.
template <bool STAGED, bool ACTIVE_CHECK>
__device__ __forceinline__ void tans_step(TansLane& d, bool active, uint32_t tbase,
                                          const uint32_t* wg, uint32_t ws, uint32_t last,
                                          uint32_t R, uint32_t lt, uint32_t ma, uint16_t* o) {
    const bool need = (!ACTIVE_CHECK || active) && d.cnt < R;
    const uint32_t m = __ballot_sync(0xFFFFFFFFu, need);
    const uint32_t q = min(d.p + __popc(m & lt), last);
    const uint32_t w = STAGED ? lds_u32(ws + 4u * q) : __ldg(wg + q);
    if (need) tans_insert(d, w);
    d.p += __popc(m);
    if (!ACTIVE_CHECK || active) tans_decode(d, lds_u32(d.xa), tbase, ma, o);
}

// Two steps of a full chunk with one word load: a lane that takes a word at a
// step holds at least 32 - 12 bits at the next one, so it takes at most one
// word per pair of steps. Its need at the second step follows from the first
// step's bit count (table entry already read), and a word it takes there may
// enter the buffer a step early: it goes above the bits the first step reads,
// and with fewer than R + 12 <= 24 bits held it fits in the 64-bit buffer. The
// second step's words follow the first step's in the shared stream. STAGED:
// no clamp; the shared-memory allocation extends far enough past the payload
// for the most words any chunk can take (16 per step).
template <bool STAGED>
__device__ __forceinline__ void tans_pair(TansLane& d, uint32_t tbase, const uint32_t* wg,
                                          uint32_t ws, uint32_t last, uint32_t R, uint32_t lt,
                                          uint32_t ma, uint16_t* o) {
    const uint32_t t0 = lds_u32(d.xa);
    const bool need0 = d.cnt < R;
    const bool need1 = !need0 && d.cnt - (t0 & 15u) < R;
    const uint32_t m0 = __ballot_sync(0xFFFFFFFFu, need0);
    const uint32_t m1 = __ballot_sync(0xFFFFFFFFu, need1);
    const uint32_t c0 = __popc(m0);
    uint32_t q = d.p + (need0 ? __popc(m0 & lt) : c0 + __popc(m1 & lt));
    if (!STAGED) q = min(q, last);
    const uint32_t w = STAGED ? lds_u32(ws + 4u * q) : __ldg(wg + q);
    if (need0 || need1) tans_insert(d, w);
    d.p += c0 + __popc(m1);
    tans_decode(d, t0, tbase, ma, o);
    tans_decode(d, lds_u32(d.xa), tbase, ma + 32u, o + 32);
}

// Decode chunk c of item I with warp `warp` (all 32 lanes).
template <int MAXI>
__device__ void tans_chunk(const TansParams<MAXI>& P, const DecodeItem& I, uint64_t c,
                           TansShared& S, int warp, int lane, uint32_t& phase) {
    const uint8_t* st = I.stream;
    const uint32_t C = I.block;
    const TansLayout L = tans_layout(I.n, C);
    const uint32_t R = S.info[0], Lst = 1u << R;
    const uint64_t E = ld_u64(st + 64);
    const uint32_t* offs = reinterpret_cast<const uint32_t*>(st + L.off_offs);
    const uint64_t start = 16ull * offs[c];
    const uint64_t end = c + 1 < L.nb ? 16ull * offs[c + 1] : E;
    const uint32_t len = uint32_t(min(uint64_t(C), I.n - c * C));
    // E lies inside the stream (header check); the chunks follow one another
    // from offset 0; a chunk payload is a whole number of 16-byte units holding
    // the 64 bytes of states and at least one word (lane 0 takes one at step 0)
    if ((c == 0 && start != 0) || start > end || end > E || end - start < 80u ||
        (end & 15u) != 0u) {
        if (lane == 0) report(P.status, kStatusCorrupt);
        return;
    }
    const uint64_t psize = end - start;
    const uint8_t* pay_g = st + L.off_exp + start;
    uint8_t* pay_s = S.stage + size_t(warp) * tans_stage_bytes(P.max_chunk);
    uint8_t* man_s = pay_s + tans_pay_stage(P.max_chunk);
    const bool staged = psize <= tans_pay_stage(C);
    const uint32_t man16 = len & ~15u;
    // stage: the payload (if it fits) and the chunk's mantissa bytes. The
    // previous chunk's reads are done and its plain stores of mantissa bytes
    // are ordered before the bulk copies that overwrite them.
    fence_proxy_async_smem();
    __syncwarp();
    if (lane == 0) {
        const uint32_t bytes = (staged ? uint32_t(psize) : 0u) + man16;
        if (bytes) {
            mbar_arrive_expect_tx(&S.bar[warp], bytes);
            if (staged) bulk_load(pay_s, pay_g, uint32_t(psize), &S.bar[warp]);
            if (man16) bulk_load(man_s, st + L.off_man + c * C, man16, &S.bar[warp]);
        } else {
            mbar_arrive(&S.bar[warp]);
        }
    }
    if (uint32_t(lane) < len - man16) man_s[man16 + lane] = st[L.off_man + c * C + man16 + lane];
    const bool ok = mbar_wait(&S.bar[warp], phase, nullptr);
    phase ^= 1u;
    __syncwarp();
    if (!__all_sync(0xFFFFFFFFu, ok)) {
        if (lane == 0) report(P.status, kStatusTimeout);
        return;
    }
    const uint8_t* pay = staged ? pay_s : pay_g;
    const uint32_t avail = uint32_t((psize - 64u) / 4u);
    const uint32_t X0 = reinterpret_cast<const uint16_t*>(pay)[lane];
    bool bad = X0 >= Lst || (uint32_t(lane) >= len && X0 != 0u);
    const uint32_t tbase = smem_addr(S.table);
    TansLane d{tbase + 4u * (X0 & (Lst - 1u)), 0u, 0u, 0u, 0u};
    const uint32_t* wg = reinterpret_cast<const uint32_t*>(pay_g + 64);
    const uint32_t ws = smem_addr(pay_s + 64);
    const uint32_t lt = lanemask_lt();
    uint32_t ma = smem_addr(man_s) + uint32_t(lane);
    uint16_t* o = I.out + c * C + lane;
    const uint32_t steps = (len + 31u) >> 5;
    if (len == C) {  // a full chunk: every lane active at every step, steps even
        if (staged) {
#pragma unroll 2
            for (uint32_t k = 0; k < steps; k += 2, ma += 64u, o += 64)
                tans_pair<true>(d, tbase, wg, ws, avail - 1u, R, lt, ma, o);
        } else {
#pragma unroll 2
            for (uint32_t k = 0; k < steps; k += 2, ma += 64u, o += 64)
                tans_pair<false>(d, tbase, wg, ws, avail - 1u, R, lt, ma, o);
        }
    } else {
        for (uint32_t k = 0; k < steps; ++k, ma += 32u, o += 32) {
            const bool active = 32u * k + uint32_t(lane) < len;
            if (staged)
                tans_step<true, true>(d, active, tbase, wg, ws, avail - 1u, R, lt, ma, o);
            else
                tans_step<false, true>(d, active, tbase, wg, ws, avail - 1u, R, lt, ma, o);
        }
    }
    // a valid chunk: every lane back at state 0 with no bits left, every word
    // read inside the payload, fewer than 4 unused words and those zero
    bad |= d.xa != tbase || (d.lo | d.hi) != 0u || d.p > avail || avail - d.p > 3u;
    if (!bad && d.p + uint32_t(lane) < avail)
        bad = reinterpret_cast<const uint32_t*>(pay + 64)[d.p + lane] != 0u;
    if (__any_sync(0xFFFFFFFFu, bad) && lane == 0) report(P.status, kStatusCorrupt);
}

template <int MAXI>
__global__ void __launch_bounds__(kTansThreads)
    tans_decode_kernel(const __grid_constant__ TansParams<MAXI> P) {
    extern __shared__ __align__(128) unsigned char smem[];
    TansShared S;
    S.table = reinterpret_cast<uint32_t*>(smem);
    S.cum = S.table + kTansTable;
    S.seen = S.cum + 260;
    S.info = S.seen + 256;
    S.bar = reinterpret_cast<unsigned long long*>(S.info + 4);
    S.stage = reinterpret_cast<uint8_t*>(S.bar + kTansWarps);
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    if (tid < kTansWarps) mbar_init(&S.bar[tid], 1);
    if (tid == 0) asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    __syncthreads();
    // a contiguous range of tiles per block, so that it changes tensors rarely
    const uint64_t total = P.tile_begin[P.count];
    const uint64_t per = (total + gridDim.x - 1) / gridDim.x;
    const uint64_t t0 = min(total, per * blockIdx.x), t1 = min(total, t0 + per);
    uint32_t cur = 0xFFFFFFFFu, phase = 0;
    for (uint64_t t = t0; t < t1; ++t) {
        const uint32_t it = tans_find_item(P, t);
        const DecodeItem& I = P.item[it];
        if (it != cur) {
            __syncthreads();  // every warp is done with the previous table
            tans_build(P, I, S);
            cur = it;
        }
        if (S.info[1] == 0) continue;  // a tensor whose header or counts are corrupt
        const uint64_t c = (t - P.tile_begin[it]) * kTansWarps + uint64_t(warp);
        if (c < tans_chunks(I.n, I.block)) tans_chunk(P, I, c, S, warp, lane, phase);
    }
}

template <int MAXI>
cudaError_t tans_launch(const DecodeItem* items, uint32_t count, int32_t* status,
                        cudaStream_t stream) {
    static_assert(sizeof(TansParams<MAXI>) <= 32000, "launch parameters exceed the limit");
    TansParams<MAXI> p;
    p.status = status;
    p.count = count;
    p.max_chunk = 0;
    uint64_t tiles = 0;
    for (uint32_t i = 0; i < count; ++i) {
        p.item[i] = items[i];
        p.tile_begin[i] = tiles;
        tiles += tans_tiles(items[i].n, items[i].block);
        p.max_chunk = max(p.max_chunk, items[i].block);
    }
    p.tile_begin[count] = tiles;
    if (tiles == 0) return cudaSuccess;
    const size_t smem = 4u * (kTansTable + 260u + 256u + 4u) + 8u * kTansWarps +
                        size_t(kTansWarps) * tans_stage_bytes(p.max_chunk) + tans_read_slack(p.max_chunk);
    static std::mutex mu;
    static int sms_of[64];
    static size_t smem_set[64];
    int dev = 0;
    cudaError_t err = cudaGetDevice(&dev);
    if (err != cudaSuccess) return err;
    if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
    {
        std::lock_guard<std::mutex> lock(mu);
        if (sms_of[dev] == 0) {
            err = cudaDeviceGetAttribute(&sms_of[dev], cudaDevAttrMultiProcessorCount, dev);
            if (err != cudaSuccess) return err;
        }
        if (smem_set[dev] < smem) {
            err = cudaFuncSetAttribute(tans_decode_kernel<MAXI>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem));
            if (err != cudaSuccess) return err;
            smem_set[dev] = smem;
        }
    }
    int per_sm = 0;
    err = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, tans_decode_kernel<MAXI>,
                                                        kTansThreads, smem);
    if (err != cudaSuccess) return err;
    const uint64_t cap = uint64_t(max(per_sm, 1)) * uint64_t(sms_of[dev]);
    const unsigned grid = unsigned(tiles < cap ? tiles : cap);
    tans_decode_kernel<MAXI><<<grid, kTansThreads, smem, stream>>>(p);
    return cudaGetLastError();
}

}  // namespace

bool tans_chunk_ok(uint32_t C) { return C == 1024 || C == 2048 || C == 4096 || C == 8192; }

uint64_t tans_fixed_bytes(uint64_t n, uint32_t C) { return tans_layout(n, C).off_exp; }

cudaError_t launch_decode_tans(const DecodeItem* items, uint32_t count, int32_t* status,
                               cudaStream_t stream) {
    constexpr uint32_t kBatch = 256;
    if (count == 1) return tans_launch<1>(items, 1, status, stream);
    for (uint32_t i = 0; i < count; i += kBatch) {
        const uint32_t c = min(kBatch, count - i);
        const cudaError_t err = tans_launch<kBatch>(items + i, c, status, stream);
        if (err != cudaSuccess) return err;
    }
    return cudaSuccess;
}

}  // namespace wc

// ===========================================================================
// Encoder: five launches per batch, none waiting on another thread block.
//   tans_hist     every tensor's exponent histogram (block-local counts, then
//                 global 64-bit adds) and its sign+mantissa plane
//   tans_plan     one block per tensor: the normalized counts (written into
//                 the stream), the header fields known before E, the zero
//                 padding of the fixed sections
//   tans_encode   one warp per chunk, twice: first only the payload sizes,
//                 then (after the scan placed every chunk) the payloads
//   tans_scan     one block per tensor: chunk offsets, E, total size
// ===========================================================================
namespace wc {
namespace {

constexpr int kEncWarps = 4;
constexpr int kEncThreads = 32 * kEncWarps;
constexpr uint32_t kHistTile = 8192;

struct TansEncItem {
    const uint16_t* in;
    uint8_t* out;
    uint64_t* out_bytes;
    uint64_t n;
    uint32_t chunk, log;        // C and R
    uint64_t chunk_begin;       // the tensor's first chunk in the batch
    uint64_t tile_begin;        // the tensor's first histogram tile in the batch
};

template <int MAXI>
struct TansEncParams {
    TansEncItem item[MAXI];
    uint64_t* hist;             // count x 256 counts
    uint32_t* sizes;            // one per chunk of the batch: payload bytes
    uint64_t total_chunks, total_tiles;
    uint32_t count, max_chunk, max_log, pass;  // pass 0: sizes only, 1: write
};

template <int MAXI>
__device__ __forceinline__ uint32_t enc_find(const TansEncParams<MAXI>& P, uint64_t u, bool chunks) {
    int lo = 0, hi = int(P.count) - 1;
    while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if ((chunks ? P.item[mid].chunk_begin : P.item[mid].tile_begin) <= u) lo = mid; else hi = mid - 1;
    }
    return uint32_t(lo);
}

template <int MAXI>
__global__ void __launch_bounds__(256) tans_hist(const __grid_constant__ TansEncParams<MAXI> P) {
    __shared__ uint32_t h[256];
    for (uint64_t t = blockIdx.x; t < P.total_tiles; t += gridDim.x) {
        const uint32_t it = enc_find(P, t, false);
        const TansEncItem& I = P.item[it];
        const uint64_t first = (t - I.tile_begin) * kHistTile;
        const uint32_t len = uint32_t(min(uint64_t(kHistTile), I.n - first));
        h[threadIdx.x] = 0;
        __syncthreads();
        const TansLayout L = tans_layout(I.n, I.chunk);
        // 32 elements per thread: their exponents counted, their sign+mantissa
        // bytes stored as two 16-byte words
        const uint32_t el = 32u * threadIdx.x;
        if (el + 32u <= len) {  // four 16-byte loads (a tile starts 16-byte aligned)
            const uint4* src = reinterpret_cast<const uint4*>(I.in + first + el);
            uint32_t sw[8];
#pragma unroll
            for (uint32_t v = 0; v < 4; ++v) {
                const uint4 a = src[v];
                uint32_t e0, e1;
                split_quad(a.x, a.y, sw[2 * v], e0);
                split_quad(a.z, a.w, sw[2 * v + 1], e1);
#pragma unroll
                for (uint32_t b = 0; b < 4; ++b) {
                    atomicAdd(&h[(e0 >> (8u * b)) & 0xFFu], 1u);
                    atomicAdd(&h[(e1 >> (8u * b)) & 0xFFu], 1u);
                }
            }
            uint8_t* dst = I.out + L.off_man + first + el;
            *reinterpret_cast<uint4*>(dst) = make_uint4(sw[0], sw[1], sw[2], sw[3]);
            *reinterpret_cast<uint4*>(dst + 16) = make_uint4(sw[4], sw[5], sw[6], sw[7]);
        } else if (el < len) {  // the ragged end of a tensor
            uint8_t* dst = I.out + L.off_man + first + el;
            for (uint32_t j = 0; el + j < len; ++j) {
                const uint32_t x = uint32_t(I.in[first + el + j]);
                atomicAdd(&h[(x >> 7) & 0xFFu], 1u);
                dst[j] = uint8_t(((x >> 8) & 0x80u) | (x & 0x7Fu));
            }
        }
        __syncthreads();
        if (h[threadIdx.x]) atomicAdd(reinterpret_cast<unsigned long long*>(&P.hist[256ull * it + threadIdx.x]),
                                      (unsigned long long)h[threadIdx.x]);
        __syncthreads();
    }
}

// One block (256 threads) per tensor.
template <int MAXI>
__global__ void __launch_bounds__(256) tans_plan(const __grid_constant__ TansEncParams<MAXI> P) {
    __shared__ unsigned long long v[256];
    __shared__ int best;
    const TansEncItem& I = P.item[blockIdx.x];
    const int tid = threadIdx.x;
    const uint32_t R = I.log, Lst = 1u << R;
    const TansLayout L = tans_layout(I.n, I.chunk);
    const uint64_t c = P.hist[256ull * blockIdx.x + tid];
    // max(1, floor(c * L / n)) for every present exponent
    uint32_t f = 0;
    if (c > 0) {
        f = uint32_t(c * Lst / I.n);
        if (f == 0) f = 1;
    }
    v[tid] = f;
    __syncthreads();
    // the sum, then the adjustments: all of a shortfall to the largest count
    // (the smaller exponent on ties); an excess taken off the largest one at a
    // time (it may change)
    for (int s = 128; s > 0; s >>= 1) {
        unsigned long long a = tid < s ? v[tid] + v[tid + s] : 0;
        __syncthreads();
        if (tid < s) v[tid] = a;
        __syncthreads();
    }
    long long diff = I.n ? (long long)Lst - (long long)v[0] : 0;
    __syncthreads();
    while (diff != 0) {
        // argmax of f with the smaller index on ties: key = f << 8 | (255 - e)
        v[tid] = (unsigned long long)f << 8 | uint32_t(255 - tid);
        __syncthreads();
        for (int s = 128; s > 0; s >>= 1) {
            unsigned long long a = 0;
            if (tid < s) a = max(v[tid], v[tid + s]);
            __syncthreads();
            if (tid < s) v[tid] = a;
            __syncthreads();
        }
        if (tid == 0) best = 255 - int(v[0] & 0xFFu);
        __syncthreads();
        if (tid == best) {
            if (diff > 0) f += uint32_t(diff); else f -= 1u;
        }
        diff = diff > 0 ? 0 : diff + 1;
        __syncthreads();
    }
    uint8_t* out = I.out;
    reinterpret_cast<uint16_t*>(out + kHeaderBytes)[tid] = uint16_t(f);
    // the header (E and the total come from the scan) and zero padding
    if (tid < 16) {
        uint64_t w = 0;
        switch (tid) {
            case 0: w = kMagic | (uint64_t(kVersion) << 32) | (uint64_t(kHeaderBytes) << 48); break;
            case 1: w = uint64_t(I.chunk) | (uint64_t(4) << 32); break;
            case 2: w = I.n; break;
            case 3: w = L.nb; break;
            case 4: w = kHeaderBytes; break;
            case 5: w = L.off_offs; break;
            case 6: w = L.off_man; break;
            case 7: w = L.off_exp; break;
            case 11: w = R; break;
            default: w = 0; break;  // 8, 9: written by the scan; 10: no low plane
        }
        if (tid != 8 && tid != 9) reinterpret_cast<uint64_t*>(out)[tid] = w;
    }
    for (uint64_t i = L.off_offs + 4 * L.nb + tid; i < L.off_man; i += 256) out[i] = 0;
    for (uint64_t i = L.off_man + I.n + tid; i < L.off_exp; i += 256) out[i] = 0;
}

// The decoding-order words of one lane that fit before this many bits.
__host__ __device__ inline uint32_t tans_lane_cap(uint32_t C, uint32_t R) {
    return 2u + (C / 32u) * R / (33u - R);
}

struct EncShared {
    uint16_t* freq;      // 256
    uint32_t* pbase;     // 256: first pos entry of each exponent
    uint32_t* seen;      // 256
    uint2* dof;          // 256: {delta, pbase - f}, see tans_enc_tables
    uint16_t* pos;       // L: state of each (exponent, occurrence)
    uint8_t* warp_area;  // per warp: C u16 (value | bits << 12), then 32 x cap words
};

// Encoding tables of item I (all threads of the block): the same spread as
// the decoder's, inverted: pos[pbase[e] + v - f[e]] = the state that decodes
// the v-th occurrence of e.
__device__ void tans_enc_tables(const TansEncItem& I, EncShared& S) {
    const int tid = threadIdx.x, lane = tid & 31;
    const uint32_t R = I.log, Lst = 1u << R;
    for (int e = tid; e < 256; e += kEncThreads)
        S.freq[e] = reinterpret_cast<const uint16_t*>(I.out + kHeaderBytes)[e];
    __syncthreads();
    if (tid < 32) {  // exclusive prefix of the counts, 8 per lane
        uint32_t loc[8], s = 0;
#pragma unroll
        for (int j = 0; j < 8; ++j) { loc[j] = s; s += S.freq[8 * lane + j]; }
        uint32_t incl = s;
        for (int d = 1; d < 32; d <<= 1) {
            const uint32_t y = __shfl_up_sync(0xFFFFFFFFu, incl, d);
            if (lane >= d) incl += y;
        }
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            S.pbase[8 * lane + j] = incl - s + loc[j];
            S.seen[8 * lane + j] = S.freq[8 * lane + j];
        }
    }
    __syncthreads();
    // Per exponent, the encoder's bit count by one add and shift: from a state
    // x in [L, 2L) it emits nb0 = R - floor(log2 f) bits, or one fewer when
    // x < f << nb0 (then x >> (nb0 - 1) < 2f already); with delta =
    // (nb0 << 16) - (f << nb0), (x + delta) >> 16 is that count (|x - (f << nb0)|
    // < L <= 2^12, mod 2^32). The next state's slot is (x >> nb) + pbase - f.
    for (int e = tid; e < 256; e += kEncThreads) {
        const uint32_t f = S.freq[e];
        const uint32_t nb0 = f ? R - (31u - __clz(f)) : 0u;
        S.dof[e] = make_uint2(f ? (nb0 << 16) - (f << nb0) : 0u, S.pbase[e] - f);
    }
    // the spread into pos (as a temporary state -> exponent map)
    const uint32_t step = (Lst >> 1) + (Lst >> 3) + 3u;
    for (uint32_t k = tid; k < Lst; k += kEncThreads) {
        int lo = 0, hi = 255;
        while (lo < hi) {
            const int mid = (lo + hi + 1) >> 1;
            if (S.pbase[mid] <= k) lo = mid; else hi = mid - 1;
        }
        S.pos[(k * step) & (Lst - 1u)] = uint16_t(lo);
    }
    __syncthreads();
    // occurrences in increasing state order (one warp), then the inverse map:
    // first into the per-warp areas as (e, v) pairs, since pos is still read
    uint32_t* tmp = reinterpret_cast<uint32_t*>(S.warp_area);
    if (tid < 32) {
        for (uint32_t x0 = 0; x0 < Lst; x0 += 32) {
            const uint32_t X = x0 + uint32_t(lane);
            const uint32_t e = S.pos[X];
            const uint32_t grp = __match_any_sync(0xFFFFFFFFu, e);
            const uint32_t v = S.seen[e] + __popc(grp & lanemask_lt());
            __syncwarp();
            if ((grp >> lane) == 1u) S.seen[e] = v + 1u;
            tmp[X] = S.pbase[e] + v - S.freq[e];
            __syncwarp();
        }
    }
    __syncthreads();
    for (uint32_t X = tid; X < Lst; X += kEncThreads) S.pos[tmp[X]] = uint16_t(X);
    __syncthreads();
}

template <int MAXI>
__global__ void __launch_bounds__(kEncThreads) tans_encode(const __grid_constant__ TansEncParams<MAXI> P) {
    extern __shared__ __align__(128) unsigned char smem[];
    EncShared S;
    S.freq = reinterpret_cast<uint16_t*>(smem);
    S.pbase = reinterpret_cast<uint32_t*>(smem + 512);
    S.seen = S.pbase + 256;
    S.dof = reinterpret_cast<uint2*>(smem + 2560);
    S.pos = reinterpret_cast<uint16_t*>(smem + 4608);
    S.warp_area = smem + 4608 + 2 * (1u << P.max_log);
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const uint32_t cap = tans_lane_cap(P.max_chunk, P.max_log);
    const size_t area = 2ull * P.max_chunk + 128ull * cap;
    uint16_t* elem = reinterpret_cast<uint16_t*>(S.warp_area + size_t(warp) * area);
    uint32_t* lw = reinterpret_cast<uint32_t*>(S.warp_area + size_t(warp) * area + 2ull * P.max_chunk) + lane * cap;
    // a contiguous range of 4-chunk groups per block
    const uint64_t groups = (P.total_chunks + kEncWarps - 1) / kEncWarps;
    const uint64_t per = (groups + gridDim.x - 1) / gridDim.x;
    const uint64_t g0 = min(groups, per * blockIdx.x), g1 = min(groups, g0 + per);
    int cur = -1;
    for (uint64_t g = g0; g < g1; ++g) {
        // a group of four chunks may span several tensors: one round per
        // tensor, in order, each warp encoding its chunk in its tensor's round
        for (uint32_t r = 0; r < uint32_t(kEncWarps); ++r) {
            const uint64_t cr = g * kEncWarps + r;
            if (cr >= P.total_chunks) break;
            const uint32_t want = enc_find(P, cr, true);
            if (r > 0 && want == enc_find(P, cr - 1, true)) continue;  // that tensor's round ran
            if (int(want) != cur) {
                __syncthreads();
                tans_enc_tables(P.item[want], S);
                cur = int(want);
            }
            const uint64_t cg = g * kEncWarps + uint64_t(warp);
            if (cg >= P.total_chunks || enc_find(P, cg, true) != uint32_t(cur)) continue;
            const TansEncItem& I = P.item[cur];
            const uint64_t c = cg - I.chunk_begin;
            const uint32_t C = I.chunk, R = I.log, Lst = 1u << R;
            const uint32_t len = uint32_t(min(uint64_t(C), I.n - c * C));
            const uint16_t* x = I.in + c * C;
            // 0. the chunk's exponents into the element area (16-byte loads of eight
            //    words each; a chunk starts 16-byte aligned), so that the serial
            //    loop below waits on shared memory, not on global loads
            for (uint32_t v = uint32_t(lane); 8u * v < len; v += 32u) {
                const uint32_t i0 = 8u * v;
                uint32_t wd[4];
                if (i0 + 8u <= len) {
                    const uint4 a = *reinterpret_cast<const uint4*>(x + i0);
                    wd[0] = a.x; wd[1] = a.y; wd[2] = a.z; wd[3] = a.w;
                } else {
#pragma unroll
                    for (uint32_t h = 0; h < 4; ++h) {
                        const uint32_t lo = i0 + 2u * h < len ? uint32_t(x[i0 + 2u * h]) : 0u;
                        const uint32_t hi = i0 + 2u * h + 1u < len ? uint32_t(x[i0 + 2u * h + 1u]) : 0u;
                        wd[h] = lo | (hi << 16);
                    }
                }
                // two words' exponents (bits 14..7 of each half) as two 16-bit lanes
                *reinterpret_cast<uint4*>(elem + i0) =
                    make_uint4((wd[0] >> 7) & 0x00FF00FFu, (wd[1] >> 7) & 0x00FF00FFu,
                               (wd[2] >> 7) & 0x00FF00FFu, (wd[3] >> 7) & 0x00FF00FFu);
            }
            __syncwarp();
            // 1. backwards: each element's bits (value | count << 12), in place of its exponent
            uint32_t st = Lst;
            const uint32_t steps = len > uint32_t(lane) ? (len - lane + 31u) >> 5 : 0u;
#pragma unroll 4
            for (uint32_t k = steps; k-- > 0;) {
                const uint32_t i = uint32_t(lane) + 32u * k;
                const uint32_t e = elem[i];
                const uint2 d = S.dof[e];
                const uint32_t nb = (st + d.x) >> 16;  // the smallest nb with (st >> nb) < 2f
                elem[i] = uint16_t((st & low_mask(nb)) | (nb << 12));
                st = Lst + S.pos[(st >> nb) + d.y];
            }
            // 2. forwards: the lane's bits packed 32 to a word
            uint32_t nw = 0, acc_bits = 0;
            uint64_t acc = 0;
            for (uint32_t k = 0; k < steps; ++k) {
                const uint32_t q = elem[uint32_t(lane) + 32u * k];
                acc |= uint64_t(q & 0xFFFu) << acc_bits;
                acc_bits += q >> 12;
                if (acc_bits >= 32u) {
                    lw[nw++] = uint32_t(acc);
                    acc >>= 32;
                    acc_bits -= 32u;
                }
            }
            if (acc_bits) lw[nw++] = uint32_t(acc);
            __syncwarp();
            // 3. the decoder's order: step by step, the lanes holding fewer than
            //    R bits take their next word (zero past the lane's bits)
            uint8_t* pay = nullptr;
            if (P.pass == 1) {
                const TansLayout Lt = tans_layout(I.n, C);
                pay = I.out + Lt.off_exp + 16ull * reinterpret_cast<const uint32_t*>(I.out + Lt.off_offs)[c];
                reinterpret_cast<uint16_t*>(pay)[lane] = uint16_t(st - Lst);
            }
            uint32_t cnt = 0, p = 0, j = 0;
            const uint32_t maxk = (len + 31u) >> 5;
            for (uint32_t k = 0; k < maxk; ++k) {
                const bool active = uint32_t(lane) + 32u * k < len;
                const bool need = active && cnt < R;
                const uint32_t m = __ballot_sync(0xFFFFFFFFu, need);
                if (need) {
                    const uint32_t w = j < nw ? lw[j] : 0u;
                    ++j;
                    if (pay) reinterpret_cast<uint32_t*>(pay + 64)[p + __popc(m & lanemask_lt())] = w;
                    cnt += 32u;
                }
                p += __popc(m);
                if (active) cnt -= elem[uint32_t(lane) + 32u * k] >> 12;
            }
            const uint32_t size = (64u + 4u * p + 15u) & ~15u;
            if (pay) {  // zero padding to 16 bytes
                const uint32_t pad_from = 64u + 4u * p;
                if (pad_from + 4u * uint32_t(lane) < size) reinterpret_cast<uint32_t*>(pay + pad_from)[lane] = 0u;
            } else if (lane == 0) {
                P.sizes[cg] = size;
            }
            __syncwarp();
        }
    }
}

// One block (1024 threads) per tensor: chunk offsets = exclusive prefix of the
// payload sizes (16-byte units), E, the header's E and total, out_bytes.
template <int MAXI>
__global__ void __launch_bounds__(1024) tans_scan(const __grid_constant__ TansEncParams<MAXI> P) {
    __shared__ unsigned long long warp_sum[32];
    __shared__ unsigned long long carry;
    const TansEncItem& I = P.item[blockIdx.x];
    const TansLayout L = tans_layout(I.n, I.chunk);
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    if (tid == 0) carry = 0;
    __syncthreads();
    uint32_t* offs = reinterpret_cast<uint32_t*>(I.out + L.off_offs);
    for (uint64_t b = 0; b < L.nb; b += 1024) {
        const uint64_t c = b + uint64_t(tid);
        const unsigned long long s = c < L.nb ? P.sizes[I.chunk_begin + c] : 0ull;
        unsigned long long incl = s;
        for (int d = 1; d < 32; d <<= 1) {
            const unsigned long long y = __shfl_up_sync(0xFFFFFFFFu, incl, d);
            if (lane >= d) incl += y;
        }
        if (lane == 31) warp_sum[warp] = incl;
        __syncthreads();
        unsigned long long before = carry;
        for (int k = 0; k < warp; ++k) before += warp_sum[k];
        if (c < L.nb) offs[c] = uint32_t((before + incl - s) >> 4);
        __syncthreads();
        if (tid == 1023) carry = before + incl;
        __syncthreads();
    }
    if (tid == 0) {
        const uint64_t E = carry;
        reinterpret_cast<uint64_t*>(I.out)[8] = E;
        reinterpret_cast<uint64_t*>(I.out)[9] = L.off_exp + E;
        *I.out_bytes = L.off_exp + E;
    }
}

template <int MAXI>
cudaError_t tans_encode_batch(const EncodeItem* items, const uint32_t* logs, uint32_t count,
                              uint8_t* ws, cudaStream_t stream) {
    static_assert(sizeof(TansEncParams<MAXI>) <= 32000, "launch parameters exceed the limit");
    TansEncParams<MAXI> p;
    memset(&p, 0, sizeof(p));
    uint64_t chunks = 0, tiles = 0;
    p.max_chunk = 1024;
    p.max_log = kTansMinLog;
    for (uint32_t i = 0; i < count; ++i) {
        TansEncItem& t = p.item[i];
        t.in = items[i].in;
        t.out = items[i].out;
        t.out_bytes = items[i].out_bytes;
        t.n = items[i].n;
        t.chunk = items[i].block;
        t.log = logs[i];
        t.chunk_begin = chunks;
        t.tile_begin = tiles;
        chunks += tans_chunks(t.n, t.chunk);
        tiles += (t.n + kHistTile - 1) / kHistTile;
        p.max_chunk = max(p.max_chunk, t.chunk);
        p.max_log = max(p.max_log, t.log);
    }
    p.count = count;
    p.total_chunks = chunks;
    p.total_tiles = tiles;
    p.hist = reinterpret_cast<uint64_t*>(ws);
    p.sizes = reinterpret_cast<uint32_t*>(ws + 2048ull * count);
    cudaError_t err = cudaMemsetAsync(p.hist, 0, 2048ull * count, stream);
    if (err != cudaSuccess) return err;
    int dev = 0, sms = 0;
    if ((err = cudaGetDevice(&dev)) != cudaSuccess) return err;
    if ((err = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess)
        return err;
    if (tiles) tans_hist<MAXI><<<unsigned((tiles < 4ull * uint64_t(sms) ? tiles : 4ull * uint64_t(sms))), 256, 0, stream>>>(p);
    tans_plan<MAXI><<<count, 256, 0, stream>>>(p);
    if (chunks) {
        const uint32_t cap = tans_lane_cap(p.max_chunk, p.max_log);
        const size_t smem = 4608 + 2ull * (1u << p.max_log) +
                            size_t(kEncWarps) * (2ull * p.max_chunk + 128ull * cap);
        if ((err = cudaFuncSetAttribute(tans_encode<MAXI>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                        int(smem))) != cudaSuccess)
            return err;
        int per_sm = 0;
        if ((err = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, tans_encode<MAXI>, kEncThreads,
                                                                 smem)) != cudaSuccess)
            return err;
        const uint64_t groups = (chunks + kEncWarps - 1) / kEncWarps;
        const unsigned grid = unsigned(groups < uint64_t(max(per_sm, 1)) * uint64_t(sms) ? groups : uint64_t(max(per_sm, 1)) * uint64_t(sms));
        p.pass = 0;
        tans_encode<MAXI><<<grid, kEncThreads, smem, stream>>>(p);
        tans_scan<MAXI><<<count, 1024, 0, stream>>>(p);
        p.pass = 1;
        tans_encode<MAXI><<<grid, kEncThreads, smem, stream>>>(p);
    } else {
        tans_scan<MAXI><<<count, 1024, 0, stream>>>(p);
    }
    return cudaGetLastError();
}

}  // namespace

uint64_t tans_bound_bytes(uint64_t n, uint32_t C, uint32_t R) {
    const TansLayout L = tans_layout(n, C);
    uint64_t worst = 0;
    for (uint64_t c = 0; c < L.nb; ++c) {
        const uint64_t len = min(uint64_t(C), n - c * C);
        const uint64_t k = (len + 31) / 32;
        worst += (64 + 4 * 32 * (1 + k * R / (33 - R)) + 15) & ~uint64_t(15);
    }
    return L.off_exp + worst;
}

uint64_t tans_workspace_bytes(const EncodeItem* items, uint32_t count) {
    uint64_t total = 0;
    for (uint32_t base = 0; base < count; base += 256) {
        const uint32_t c = min(256u, count - base);
        uint64_t chunks = 0;
        for (uint32_t i = 0; i < c; ++i) chunks += tans_chunks(items[base + i].n, items[base + i].block);
        total += (2048ull * c + 4 * chunks + 15) & ~uint64_t(15);
    }
    return total;
}

cudaError_t launch_encode_tans(const EncodeItem* items, const uint32_t* logs, uint32_t count,
                               void* workspace, cudaStream_t stream) {
    uint8_t* ws = static_cast<uint8_t*>(workspace);
    for (uint32_t base = 0; base < count; base += 256) {
        const uint32_t c = min(256u, count - base);
        const cudaError_t err = c == 1 ? tans_encode_batch<1>(items + base, logs + base, 1, ws, stream)
                                       : tans_encode_batch<256>(items + base, logs + base, c, ws, stream);
        if (err != cudaSuccess) return err;
        uint64_t chunks = 0;
        for (uint32_t i = 0; i < c; ++i) chunks += tans_chunks(items[base + i].n, items[base + i].block);
        ws += (2048ull * c + 4 * chunks + 15) & ~uint64_t(15);
    }
    return cudaSuccess;
}

}  // namespace wc
