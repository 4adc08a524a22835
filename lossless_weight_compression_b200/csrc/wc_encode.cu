// wc_encode.cu -- single-pass WCB1 encoder for sm_100a.
//
// Every step of the encoding of "ENEC: A Lossless AI Model Compression Method
// Enabling Fast Inference on Ascend NPUs", Abstract, runs in one pass over
// 8192-element tiles (whole blocks of B elements):
//   split      each BF16 word -> exponent byte e, sign+mantissa byte s
//   width      per block lo = min e, hi = max e, w = bits(hi - lo); raw
//              fallback (base 0) when w == 8, else base = lo
//   scan       exclusive prefix sum of the block sizes ceil(L/8)*w: inside a
//              tile by a warp scan, across tiles by a decoupled look-back
//              (Merrill & Garland, "Single-pass Parallel Prefix Scan with
//              Decoupled Look-back", 2016) over per-tile state words
//   remap+pack v = e - base, packed by hierarchical halving (pairs, quads,
//              octets) into w bytes per octet
// The input is read once.
//
// The kernel is persistent and warp-specialised; each thread block runs
//   a producer warp   takes the next tile from an atomic ticket (so a tile
//                     only ever waits on tiles that started before it), finds
//                     its tensor, and bulk-copies (cp.async.bulk) the tile's
//                     16 KB of input into one of two input stages;
//   8 worker warps    split (the mantissa bytes go straight to global memory
//                     with coalesced 16-byte stores: their position needs no
//                     prefix), reduce per-block min/max, compute widths and
//                     the tile-local scan, publish the tile's byte count at
//                     once, and pack the exponent payload into one of four
//                     output stages -- none of this waits on other tiles;
//   2 store warps     take alternate tiles; each runs the look-back over a
//                     256-tile window per round trip (wide enough to keep up
//                     with the rate at which tiles start), publishes the
//                     inclusive prefix, writes the block headers and offsets,
//                     bulk-stores the exponent payload at its offset and, for
//                     a tensor's last tile, the container header and padding.
//                     Several store warps keep look-back latency off the
//                     workers' critical path.
// Stages are handed over with mbarriers; every wait is bounded by the device
// timer, and a tile whose look-back gives up marks its state word so that
// later tiles stop waiting too (WC_ERR_TIMEOUT).
#include <mutex>
#include <type_traits>

#include "wc_pack_core.cuh"

namespace wc {
namespace {

constexpr int kWorkerWarps = kThreads / 32;  // 8
constexpr int kProducerWarp = kWorkerWarps;
constexpr int kStoreWarps = 2;                // tile i goes to store warp i % 2
constexpr int kFirstStoreWarp = kWorkerWarps + 1;
constexpr int kEncodeThreads = kThreads + 32 + 32 * kStoreWarps;  // 352
constexpr int kInStages = 2;
constexpr int kOutStages = 4;
constexpr int kWindowRows = 8;  // look-back window: 8 x 32 tiles per round trip

constexpr unsigned long long kFlagAggregate = 1ull << 62;  // value = this tile's bytes
constexpr unsigned long long kFlagPrefix = 2ull << 62;     // value = bytes up to and incl. this tile
constexpr unsigned long long kFlagError = 3ull << 62;      // the tile gave up
constexpr unsigned long long kValueMask = (1ull << 62) - 1;

template <int MAXI>
struct EncodeParams {
    int32_t* status;
    uint32_t* control;          // [0] ticket counter, [1] error flag
    unsigned long long* state;  // one look-back word per tile of the batch
    uint64_t timeout_ns;
    uint64_t total_tiles;
    uint32_t count;
    uint32_t first_ticket;
    uint64_t tile_begin[MAXI + 1];  // first tile of each tensor; [count] = total
    EncodeItem item[MAXI];
};

struct __align__(16) InInfo {
    uint64_t t, lt;    // batch tile index, tile index within its tensor
    uint64_t man_off;  // byte offset of the tile's mantissa bytes in its stream
    uint64_t low_off;  // FP32: byte offset of the tile's low halves in its stream
    uint32_t item, tile_n, end, pad;
};

// F32: the tile's input is FP32 words; their high halves go through the same
// path as BF16 words and their low halves straight to the stream's low plane.
template <bool F32>
struct __align__(16) InStage {
    typename std::conditional<F32, uint32_t, uint16_t>::type words[kTile];
    InInfo info;
};

struct __align__(16) OutInfo {
    uint64_t t, lt;
    uint32_t item, tile_n, nblk, total, end, pad[3];
};

struct __align__(16) OutStage {
    uint8_t exp[kTile + 16];
    uint32_t blk[kMaxBlocksPerTile];  // base | w << 8 | tile-local payload offset << 16
    OutInfo info;
};

template <bool F32>
struct EncodeSmem {
    InStage<F32> in[kInStages];
    OutStage out[kOutStages];
    unsigned long long in_full[kInStages], in_empty[kInStages];
    unsigned long long out_full[kOutStages], out_empty[kOutStages];
    int lo[3][kMaxBlocksPerTile], hi[3][kMaxBlocksPerTile];  // per-block min/max, tile i uses i % 3
    int abort;        // some warp gave up: every wait of the block stops
    int worker_stop;  // written by workers only, before their agreement barrier
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

__device__ __forceinline__ uint32_t log2_of(uint32_t B) { return uint32_t(__ffs(int(B))) - 1u; }

// Per 16-bit lane minimum / maximum (native on sm_90 and later).
__device__ __forceinline__ uint32_t min_u16x2(uint32_t a, uint32_t b) {
    uint32_t d;
    asm("min.u16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
    return d;
}

__device__ __forceinline__ uint32_t max_u16x2(uint32_t a, uint32_t b) {
    uint32_t d;
    asm("max.u16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
    return d;
}

template <int MAXI>
__device__ __forceinline__ uint32_t find_item(const EncodeParams<MAXI>& P, uint64_t t) {
    if (MAXI == 1) return 0;
    int lo = 0, hi = int(P.count) - 1;
    while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (P.tile_begin[mid] <= t) lo = mid; else hi = mid - 1;
    }
    return uint32_t(lo);
}

// The 8 worker warps meet on hardware barrier 1 (the other warps never use
// it), once per tile. Every worker reaches it on every path through an
// iteration -- a failed wait or the end of the work included -- and only then
// decides to leave, so no worker can wait there for one that has left.
__device__ __forceinline__ void workers_sync() {
    asm volatile("bar.sync 1, %0;" ::"n"(kThreads) : "memory");
}

template <bool F32>
__device__ __forceinline__ void give_up(EncodeSmem<F32>& sm, int32_t* status, int lane) {
    if (lane == 0) {
        report(status, kStatusTimeout);
        sm.abort = 1;
    }
}

// ---------------------------------------------------------------------------
// producer warp
// ---------------------------------------------------------------------------
template <int MAXI, bool F32>
__device__ void encode_produce(const EncodeParams<MAXI>& P, EncodeSmem<F32>& sm, int lane) {
    int issued_round[kInStages];  // last round whose bulk copy was issued, per stage
    for (int s = 0; s < kInStages; ++s) issued_round[s] = -1;
    // The next tile's ticket is taken while the current tile's copy is in flight,
    // so the atomic's round trip stays off the stage's critical path.
    uint64_t t_next = 0;
    if (lane == 0) t_next = uint64_t(atomicAdd(&P.control[0], 1u)) + P.first_ticket;
    t_next = __shfl_sync(0xFFFFFFFFu, t_next, 0);
    for (uint32_t i = 0;; ++i) {
        const int s = int(i % kInStages);
        const uint32_t round = i / kInStages;
        if (round > 0 && !mbar_wait(&sm.in_empty[s], (round & 1u) ^ 1u, &sm.abort, 256)) {
            give_up(sm, P.status, lane);
            break;
        }
        InStage<F32>& st = sm.in[s];
        const uint64_t t = t_next;
        if (t >= P.total_tiles) {
            if (lane == 0) {
                st.info.end = 1;
                mbar_arrive(&sm.in_full[s]);
            }
            return;
        }
        const uint32_t it = find_item(P, t);
        const EncodeItem& I = P.item[it];
        const uint64_t lt = t - P.tile_begin[it];
        const uint64_t first = lt * kTile;
        const uint32_t tile_n = I.n ? uint32_t(min(uint64_t(kTile), I.n - first)) : 0u;
        constexpr uint32_t kWordBytes = F32 ? 4u : 2u;
        const uint32_t b16 = (kWordBytes * tile_n) & ~15u;  // bytes the bulk copy can move
        const uint32_t rem = tile_n - b16 / kWordBytes;     // trailing elements loaded plainly
        using Word = typename std::conditional<F32, uint32_t, uint16_t>::type;
        const Word* in_words = reinterpret_cast<const Word*>(I.in);
        if (uint32_t(lane) < rem)
            st.words[b16 / kWordBytes + lane] = in_words[first + b16 / kWordBytes + lane];
        if (lane == 0) {
            const Layout L = make_layout(I.n, I.block, F32);
            st.info = InInfo{t, lt, L.off_man + first, L.off_low + 2 * first, it, tile_n, 0u, 0u};
        }
        __syncwarp();
        if (lane == 0) {
            if (b16) {
                mbar_arrive_expect_tx(&sm.in_full[s], b16);
                bulk_load(st.words, in_words + first, b16, &sm.in_full[s]);
                issued_round[s] = int(round);
            } else {
                mbar_arrive(&sm.in_full[s]);
            }
            t_next = uint64_t(atomicAdd(&P.control[0], 1u)) + P.first_ticket;
        }
        t_next = __shfl_sync(0xFFFFFFFFu, t_next, 0);
    }
    // Giving up: wait (bounded) for this warp's copies still in flight into shared memory.
    if (lane == 0)
        for (int s = 0; s < kInStages; ++s)
            if (issued_round[s] >= 0) mbar_wait(&sm.in_full[s], uint32_t(issued_round[s]) & 1u, nullptr);
}

// ---------------------------------------------------------------------------
// worker warps
// ---------------------------------------------------------------------------
template <int MAXI, bool F32>
__device__ void encode_work(const EncodeParams<MAXI>& P, EncodeSmem<F32>& sm, int tid, int lane,
                            int warp) {
    for (uint32_t i = 0;; ++i) {
        const int s = int(i % kInStages), o = int(i % kOutStages);
        const uint32_t rin = i / kInStages, rout = i / kOutStages;
        const bool ok = mbar_wait(&sm.in_full[s], rin & 1u, &sm.abort) &&
                        (rout == 0 || mbar_wait(&sm.out_empty[o], (rout & 1u) ^ 1u, &sm.abort));
        if (!ok) {
            give_up(sm, P.status, lane);
            if (lane == 0) sm.worker_stop = 1;
        }
        const InStage<F32>& in = sm.in[s];
        OutStage& out = sm.out[o];
        InInfo info = in.info;
        if (!ok) info.end = 0, info.tile_n = 0;
        int* lo_of = sm.lo[i % 3];
        int* hi_of = sm.hi[i % 3];
        if (info.end) {  // pass the end on to every store warp (the next kStoreWarps stages)
            for (uint32_t q = 0; q < kStoreWarps; ++q) {
                const uint32_t iq = i + q;
                const int oq = int(iq % kOutStages);
                const uint32_t rq = iq / kOutStages;
                if (q > 0 && rq > 0 && !mbar_wait(&sm.out_empty[oq], (rq & 1u) ^ 1u, &sm.abort)) {
                    give_up(sm, P.status, lane);
                    break;
                }
                if (tid == 0) sm.out[oq].info.end = 1;
                __syncwarp();
                if (lane == 0) mbar_arrive(&sm.out_full[oq]);
            }
        }
        const EncodeItem& I = P.item[info.item];
        const uint32_t B = I.block, log2B = log2_of(B), tile_n = info.end ? 0u : info.tile_n;
        const uint32_t group = min(B / kChunk, 32u);  // chunks of one block inside a warp
        const uint64_t man_base = info.man_off;

        // ---- read the input, release the input stage --------------------------------
        uint32_t x[kChunksPerThread][8];
        uint32_t nval[kChunksPerThread];
#pragma unroll
        for (int k = 0; k < kChunksPerThread; ++k) {
            const uint32_t el = uint32_t(tid + k * kThreads) * kChunk;
            const uint32_t nv = el < tile_n ? min(uint32_t(kChunk), tile_n - el) : 0u;
            nval[k] = nv;
            if (nv) {
                if (F32) {
                    // high halves into x (as BF16 pairs); low halves straight to the
                    // low plane (past the end: zeros, the plane's padding)
                    uint32_t lw[8];
#pragma unroll
                    for (int q = 0; q < 4; ++q) {
                        const uint4 a = *reinterpret_cast<const uint4*>(in.words + el + 4 * q);
                        x[k][2 * q] = prmt(a.x, a.y, 0x7632u);
                        x[k][2 * q + 1] = prmt(a.z, a.w, 0x7632u);
                        lw[2 * q] = prmt(a.x, a.y, 0x5410u);
                        lw[2 * q + 1] = prmt(a.z, a.w, 0x5410u);
                    }
                    if (nv < kChunk) {
#pragma unroll
                        for (int j = 0; j < 8; ++j) {
                            const uint32_t keep = (2u * j + 1 < nv) ? 0xFFFFFFFFu
                                                  : (2u * j < nv) ? 0x0000FFFFu : 0u;
                            lw[j] &= keep;
                        }
                    }
                    const EncodeItem& Iw = P.item[info.item];
                    uint8_t* lo_dst = Iw.out + info.low_off + 2 * el;
                    st_stream_v4(lo_dst, make_uint4(lw[0], lw[1], lw[2], lw[3]));
                    st_stream_v4(lo_dst + 16, make_uint4(lw[4], lw[5], lw[6], lw[7]));
                } else {
                    const uint4 a = *reinterpret_cast<const uint4*>(in.words + el);
                    const uint4 b = *reinterpret_cast<const uint4*>(in.words + el + 8);
                    x[k][0] = a.x; x[k][1] = a.y; x[k][2] = a.z; x[k][3] = a.w;
                    x[k][4] = b.x; x[k][5] = b.y; x[k][6] = b.z; x[k][7] = b.w;
                }
                if (nv < kChunk) {
                    // lanes past the end repeat the first element: min and max stay put
                    const uint32_t first = x[k][0] & 0xFFFFu;
#pragma unroll
                    for (int j = 0; j < 8; ++j) {
                        const uint32_t lo = (2u * j < nv) ? (x[k][j] & 0xFFFFu) : first;
                        const uint32_t hi = (2u * j + 1 < nv) ? (x[k][j] >> 16) : first;
                        x[k][j] = lo | (hi << 16);
                    }
                }
            } else {
#pragma unroll
                for (int j = 0; j < 8; ++j) x[k][j] = 0;
            }
        }
        __syncwarp();
        if (ok && !info.end && lane == 0) mbar_arrive(&sm.in_empty[s]);

        // ---- split: mantissa bytes to global memory, exponents kept; per-block min/max
        // The exponent is the top byte of a word's 15-bit magnitude, so the
        // minimum and maximum exponent are those of the smallest and largest
        // magnitude, found with 16-bit lane min/max on the sign-cleared words.
        uint32_t E[kChunksPerThread][4];
#pragma unroll
        for (int k = 0; k < kChunksPerThread; ++k) {
            const uint32_t el = uint32_t(tid + k * kThreads) * kChunk;
            const uint32_t nv = nval[k];
            uint32_t S[4];
#pragma unroll
            for (int j = 0; j < 4; ++j) split_quad(x[k][2 * j], x[k][2 * j + 1], S[j], E[k][j]);
            if (nv < kChunk) {  // mantissa bytes past the end are the plane's zero padding
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    const int valid = int(nv) - 4 * j;
                    if (valid < 4) S[j] &= valid <= 0 ? 0u : (0xFFFFFFFFu >> (32 - 8 * valid));
                }
            }
            if (nv)
                st_stream_v4(I.out + man_base + el, make_uint4(S[0], S[1], S[2], S[3]));
            // key = largest doubled magnitude << 16 | (0xFFFF - smallest): one
            // 16-bit lane maximum reduces both across the lanes of a block. x + x
            // doubles both halves' magnitudes at once: the low half's sign bit
            // moves into bit 0 of the high half, below its exponent (bits 8..15
            // of a doubled half), and the high half's sign bit leaves the word.
            uint32_t key = 0u;
            if (nv) {
                uint32_t mn = x[k][0] + x[k][0], mx = mn;
#pragma unroll
                for (int j = 1; j < 8; ++j) {
                    const uint32_t m = x[k][j] + x[k][j];
                    mn = min_u16x2(mn, m);
                    mx = max_u16x2(mx, m);
                }
                key = (max(mx & 0xFFFFu, mx >> 16) << 16) | (0xFFFFu - min(mn & 0xFFFFu, mn >> 16));
            }
            if (group == 32) {  // B >= 512: the warp's 32 chunks are one block
                key = (__reduce_max_sync(0xFFFFFFFFu, key >> 16) << 16) |
                      __reduce_max_sync(0xFFFFFFFFu, key & 0xFFFFu);
            } else {
                for (uint32_t off = 1; off < group; off <<= 1)
                    key = max_u16x2(key, __shfl_xor_sync(0xFFFFFFFFu, key, off));
            }
            const uint32_t lo = (0xFFFFu - (key & 0xFFFFu)) >> 8, hi = key >> (16 + 8);
            if ((lane & (group - 1)) == 0 && nv) {
                atomicMin(&lo_of[el >> log2B], int(lo));
                atomicMax(&hi_of[el >> log2B], int(hi));
            }
        }
        // The one barrier of the tile: all per-block min/max are in, and the workers
        // agree whether to go on. worker_stop is written only before this barrier
        // and every worker reaches it on every path, so all read the same value.
        workers_sync();
        if (sm.worker_stop || info.end) return;

        // ---- every worker warp: widths, sizes and the tile-local scan (each warp
        //      needs the offsets of its own blocks; computing them in every warp
        //      saves a barrier); worker warp 0 also publishes the tile --------------
        const uint32_t nblk = (tile_n + B - 1) >> log2B;
        uint32_t sz[2], hdr[2];
#pragma unroll
        for (int j = 0; j < 2; ++j) {
            const uint32_t b = 2 * lane + j;
            sz[j] = 0;
            hdr[j] = 0;
            if (b < nblk) {
                const uint32_t lo = lo_of[b], hi = hi_of[b], d = hi - lo;
                const uint32_t w = d ? 32u - __clz(d) : 0u;
                const uint32_t base = (w == 8u) ? 0u : lo;
                const uint32_t len = min(B, tile_n - b * B);
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
        // block b's entry lives in lane b/2, slot b&1
        const uint32_t blk_a = hdr[0] | (excl << 16), blk_b = hdr[1] | ((excl + sz[0]) << 16);
        if (warp == 0) {
            if (2 * lane < nblk) out.blk[2 * lane] = blk_a;
            if (2 * lane + 1 < nblk) out.blk[2 * lane + 1] = blk_b;
            const uint32_t total = __shfl_sync(0xFFFFFFFFu, incl, 31);
            if (lane == 0) {
                out.info = OutInfo{info.t, info.lt, info.item, tile_n, nblk, total, 0u, {0u, 0u, 0u}};
                // the first tile of a tensor knows its prefix (0); others publish their size
                store_state(&P.state[info.t], (info.lt == 0 ? kFlagPrefix : kFlagAggregate) | total);
            }
        }
        // Tile i - 1's min/max (buffer (i + 2) % 3) were read by every warp before
        // this tile's barrier; reset them now. The next tile to use that buffer,
        // i + 2, adds to it only after the barrier of tile i + 1, which this warp
        // reaches after the reset.
        if (warp == 1) {
            int* lo_next = sm.lo[(i + 2) % 3];
            int* hi_next = sm.hi[(i + 2) % 3];
            lo_next[lane] = 255;
            lo_next[lane + 32] = 255;
            hi_next[lane] = 0;
            hi_next[lane + 32] = 0;
        }

        // ---- remap and pack into the stage -----------------------------------------
#pragma unroll
        for (int k = 0; k < kChunksPerThread; ++k) {
            const uint32_t nv = nval[k];
            const uint32_t el = uint32_t(tid + k * kThreads) * kChunk;
            // block el/B's entry sits in lane (el/B)/2 (every lane takes part in the shuffles)
            const uint32_t bl = (el >> log2B) & (kMaxBlocksPerTile - 1);
            const uint32_t ea = __shfl_sync(0xFFFFFFFFu, blk_a, bl >> 1);
            const uint32_t eb = __shfl_sync(0xFFFFFFFFu, blk_b, bl >> 1);
            if (nv == 0) continue;
            const uint32_t blk = (bl & 1u) ? eb : ea;
            const uint32_t base = blk & 0xFFu, w = (blk >> 8) & 0xFFu;
            const uint32_t dst = (blk >> 16) + ((el & (B - 1)) >> 3) * w;
            uint32_t V[4];
#pragma unroll
            for (int j = 0; j < 4; ++j) V[j] = E[k][j] - base * 0x01010101u;  // e >= base: no borrows
            if (nv < kChunk) {  // lanes past the end pack as 0
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    const int valid = int(nv) - 4 * j;
                    if (valid < 4) V[j] &= valid <= 0 ? 0u : (0xFFFFFFFFu >> (32 - 8 * valid));
                }
            }
            if (nv == kChunk)
                pack_chunk_w(w, V, out.exp + dst);
            else
                pack_chunk_tail(w, V, out.exp + dst, (nv > 8 ? 2u : 1u) * w);
        }
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) mbar_arrive(&sm.out_full[o]);
    }
}

// ---------------------------------------------------------------------------
// store warp
// ---------------------------------------------------------------------------
// Decoupled look-back for tile t (index lt in its tensor): the bytes of all
// earlier tiles of the tensor. While the nearest predecessors are plain
// aggregates it reads 8 x 32 state words per round trip; while it waits on an
// unpublished predecessor it polls only the 32 nearest, backing off.
template <int MAXI>
__device__ int lookback(const EncodeParams<MAXI>& P, uint64_t t, uint64_t lt, int lane,
                        volatile int* abort, unsigned long long* prefix_out) {
    const long long first = (long long)(t - lt);  // the tensor's first tile: always a prefix
    long long top = (long long)t - 1;             // nearest tile not yet accounted for
    unsigned long long acc = 0;
    int rows = 1;
    uint32_t backoff = 32;
    const uint64_t t0 = __shfl_sync(0xFFFFFFFFu, global_timer_ns(), 0);
    while (true) {
        unsigned long long v[kWindowRows];
#pragma unroll
        for (int k = 0; k < kWindowRows; ++k) {
            const long long idx = top - (32 * k + lane);
            v[k] = (k < rows && idx >= first) ? load_state(&P.state[idx]) : kFlagPrefix;
        }
        // nearest tile (smallest distance 32k + lane) that is not a plain aggregate
        int found = -1;
        uint32_t fflag = 0;
#pragma unroll
        for (int k = 0; k < kWindowRows; ++k) {
            const unsigned b = __ballot_sync(0xFFFFFFFFu, k < rows && uint32_t(v[k] >> 62) != 1u);
            if (found < 0 && b) {
                const int l = __ffs(int(b)) - 1;
                found = 32 * k + l;
                fflag = __shfl_sync(0xFFFFFFFFu, uint32_t(v[k] >> 62), l);
            }
        }
        // everything nearer than `found` is an aggregate: account for it now
        const int upto = found < 0 ? 32 * rows : (fflag == 2u ? found + 1 : found);
        unsigned long long sum = 0;
#pragma unroll
        for (int k = 0; k < kWindowRows; ++k)
            if (32 * k + lane < upto) sum += v[k] & kValueMask;
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) sum += __shfl_xor_sync(0xFFFFFFFFu, sum, off);
        acc += sum;
        top -= upto;
        if (fflag == 2u && found >= 0) {
            *prefix_out = acc;
            return 0;
        }
        if (found < 0) {  // a full window of aggregates: read further back, wider
            rows = kWindowRows;
            continue;
        }
        if (fflag == 3u) return kStatusCorrupt;  // a predecessor gave up (already reported)
        // the nearest unaccounted predecessor has not published yet: wait, bounded
        const int stop = __shfl_sync(
            0xFFFFFFFFu,
            int(*abort || load_flag(&P.control[1]) != 0 || global_timer_ns() - t0 > P.timeout_ns),
            0);
        if (stop) return kStatusTimeout;
        __nanosleep(backoff);
        backoff = min(backoff * 2u, 1024u);
        rows = 1;
    }
}

__device__ void write_container(uint8_t* out, const Layout& L, uint64_t E, int lane) {
    if (lane < 16) {
        uint64_t v = 0;
        switch (lane) {
            case 0: v = kMagic | (uint64_t(kVersion) << 32) | (uint64_t(kHeaderBytes) << 48); break;
            case 1: v = L.block | (uint64_t(L.flags) << 32); break;  // flags: bit 0 = FP32
            case 2: v = L.n; break;
            case 3: v = L.nb; break;
            case 4: v = L.off_hdr; break;
            case 5: v = L.off_offs; break;
            case 6: v = L.off_man; break;
            case 7: v = L.off_exp; break;
            case 8: v = E; break;
            case 9: v = L.off_exp + E; break;
            case 10: v = L.off_low; break;
            default: v = 0; break;
        }
        reinterpret_cast<uint64_t*>(out)[lane] = v;
    }
}

// Zero the padding after the header, offset, mantissa and low sections. The
// bytes [n, round16(n)) of the mantissa plane and [2n, 2 round16(n)) of the
// low plane were stored as zeros by the last tile.
__device__ void write_padding(uint8_t* out, const Layout& L, int lane) {
    const uint64_t n16 = (L.n + 15) & ~uint64_t(15);
    const uint64_t a0 = L.off_hdr + 2 * L.nb, a1 = L.off_offs + 4 * L.nb;
    const uint64_t a2 = L.off_man + n16;
    const uint64_t man_end = L.fp32 ? L.off_low : L.off_exp;
    for (uint64_t i = a0 + lane; i < L.off_offs; i += 32) out[i] = 0;
    for (uint64_t i = a1 + lane; i < L.off_man; i += 32) out[i] = 0;
    for (uint64_t i = a2 + lane; i < man_end; i += 32) out[i] = 0;
    if (L.fp32)
        for (uint64_t i = L.off_low + 2 * n16 + lane; i < L.off_exp; i += 32) out[i] = 0;
}

template <int MAXI, bool F32>
__device__ void encode_store(const EncodeParams<MAXI>& P, EncodeSmem<F32>& sm, int lane, int which) {
    for (uint32_t i = uint32_t(which);; i += kStoreWarps) {
        const int o = int(i % kOutStages);
        const uint32_t round = i / kOutStages;
        if (!mbar_wait(&sm.out_full[o], round & 1u, &sm.abort, 1024)) {
            give_up(sm, P.status, lane);
            break;
        }
        const OutStage& st = sm.out[o];
        const OutInfo info = st.info;
        if (info.end) break;
        const EncodeItem& I = P.item[info.item];
        const Layout L = make_layout(I.n, I.block, F32);
        const uint64_t first = info.lt * kTile;
        const bool last_tile = info.lt + 1 == encode_tiles(I.n);

        unsigned long long prefix = 0;
        int rc = 0;
        if (info.lt > 0 && load_flag(&P.control[1]) == 0) {
            rc = lookback(P, info.t, info.lt, lane, &sm.abort, &prefix);
        } else if (info.lt > 0) {
            rc = kStatusCorrupt;  // an earlier failure: stop here without waiting
        }
        if (rc == 0) {
            if (lane == 0 && info.lt > 0)
                store_state(&P.state[info.t], kFlagPrefix | (prefix + info.total));
            const uint64_t b0 = first >> L.log2_block;
            for (uint32_t b = lane; b < info.nblk; b += 32) {
                const uint32_t blk = st.blk[b];
                reinterpret_cast<uint16_t*>(I.out + L.off_hdr)[b0 + b] = uint16_t(blk & 0xFFFFu);
                reinterpret_cast<uint32_t*>(I.out + L.off_offs)[b0 + b] =
                    uint32_t((prefix + (blk >> 16)) >> 4);
            }
            const uint32_t t16 = info.total & ~15u, rem = info.total - t16;
            uint8_t* dst = I.out + L.off_exp + prefix;  // 16-byte aligned: earlier tiles are full
            if (lane == 0 && t16) bulk_store(dst, st.exp, t16);
            if (uint32_t(lane) < rem) dst[t16 + lane] = st.exp[t16 + lane];
            if (last_tile) {
                const uint64_t E = prefix + info.total;
                write_container(I.out, L, E, lane);
                write_padding(I.out, L, lane);
                if (lane == 0) *I.out_bytes = L.off_exp + E;
            }
        } else {
            if (lane == 0) {
                store_state(&P.state[info.t], kFlagError);
                atomicExch(&P.control[1], 1u);
                if (rc == kStatusTimeout) report(P.status, kStatusTimeout);
                if (last_tile) *I.out_bytes = 0;
            }
        }
        // The stage is free once the bulk store has read it.
        if (lane == 0) {
            bulk_commit();
            bulk_wait_read<0>();
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&sm.out_empty[o]);
    }
    if (lane == 0) bulk_wait_all();
}

template <int MAXI, bool F32>
__global__ void __launch_bounds__(kEncodeThreads, F32 ? 2 : 3)
    encode_kernel(const __grid_constant__ EncodeParams<MAXI> P) {
    extern __shared__ __align__(128) unsigned char smem_raw[];
    EncodeSmem<F32>& sm = *reinterpret_cast<EncodeSmem<F32>*>(smem_raw);
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    if (tid == 0) {
        for (int s = 0; s < kInStages; ++s) {
            mbar_init(&sm.in_full[s], 1);
            mbar_init(&sm.in_empty[s], kWorkerWarps);
        }
        for (int o = 0; o < kOutStages; ++o) {
            mbar_init(&sm.out_full[o], kWorkerWarps);
            mbar_init(&sm.out_empty[o], 1);
        }
        sm.abort = 0;
        sm.worker_stop = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    if (tid < 3 * kMaxBlocksPerTile) {
        sm.lo[tid >> 6][tid & 63] = 255;
        sm.hi[tid >> 6][tid & 63] = 0;
    }
    __syncthreads();
    if (warp == kProducerWarp)
        encode_produce<MAXI, F32>(P, sm, lane);
    else if (warp >= kFirstStoreWarp)
        encode_store<MAXI, F32>(P, sm, lane, warp - kFirstStoreWarp);
    else
        encode_work<MAXI, F32>(P, sm, tid, lane, warp);
}

template <int MAXI, bool F32>
cudaError_t encode_grid(uint64_t tiles, unsigned* grid) {
    static std::mutex mu;
    static int per_device[64];
    int dev = 0;
    cudaError_t err = cudaGetDevice(&dev);
    if (err != cudaSuccess) return err;
    if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
    std::lock_guard<std::mutex> lock(mu);
    if (per_device[dev] == 0) {
        err = cudaFuncSetAttribute(encode_kernel<MAXI, F32>,
                                   cudaFuncAttributeMaxDynamicSharedMemorySize,
                                   int(sizeof(EncodeSmem<F32>)));
        if (err != cudaSuccess) return err;
        int sms = 0, per_sm = 0;
        err = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
        if (err != cudaSuccess) return err;
        err = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, encode_kernel<MAXI, F32>,
                                                            kEncodeThreads, sizeof(EncodeSmem<F32>));
        if (err != cudaSuccess) return err;
        per_device[dev] = (per_sm > 0 ? per_sm : 1) * sms;
    }
    const uint64_t cap = uint64_t(per_device[dev]);
    *grid = unsigned(tiles < cap ? tiles : cap);
    return cudaSuccess;
}

template <int MAXI, bool F32>
cudaError_t encode_batch(const EncodeItem* items, uint32_t count, uint8_t* workspace,
                         int32_t* status, uint64_t timeout_ns, uint32_t first_ticket,
                         cudaStream_t stream) {
    static_assert(sizeof(EncodeParams<MAXI>) <= 32000, "launch parameters exceed the limit");
    EncodeParams<MAXI> p;
    p.status = status;
    p.control = reinterpret_cast<uint32_t*>(workspace);
    p.state = reinterpret_cast<unsigned long long*>(workspace + 16);
    p.timeout_ns = timeout_ns;
    p.count = count;
    p.first_ticket = first_ticket;
    uint64_t tiles = 0;
    for (uint32_t i = 0; i < count; ++i) {
        p.tile_begin[i] = tiles;
        p.item[i] = items[i];
        tiles += encode_tiles(items[i].n);
    }
    p.tile_begin[count] = tiles;
    p.total_tiles = tiles;
    if (tiles == 0) return cudaSuccess;
    if (tiles >= (1ull << 31)) return cudaErrorInvalidValue;  // the ticket is 32-bit
    cudaError_t err = cudaMemsetAsync(workspace, 0, encode_workspace_bytes(tiles), stream);
    if (err != cudaSuccess) return err;
    unsigned grid = 0;
    err = encode_grid<MAXI, F32>(tiles, &grid);
    if (err != cudaSuccess) return err;
    encode_kernel<MAXI, F32><<<grid, kEncodeThreads, sizeof(EncodeSmem<F32>), stream>>>(p);
    return cudaGetLastError();
}

}  // namespace

constexpr uint32_t kEncodeBatchMax = 512;

cudaError_t launch_encode(const EncodeItem* items, uint32_t count, void* workspace,
                          int32_t* status, uint64_t timeout_ns, uint32_t first_ticket,
                          cudaStream_t stream, bool fp32) {
    uint8_t* ws = static_cast<uint8_t*>(workspace);
    if (fp32) {  // FP32 tensors: one per call
        if (count != 1) return cudaErrorInvalidValue;
        return encode_batch<1, true>(items, 1, ws, status, timeout_ns, first_ticket, stream);
    }
    if (count == 1)
        return encode_batch<1, false>(items, 1, ws, status, timeout_ns, first_ticket, stream);
    // Larger batches go out in launches of up to 512 tensors; each launch has
    // its own part of the workspace, so they can follow each other on the stream.
    for (uint32_t i = 0; i < count; i += kEncodeBatchMax) {
        const uint32_t c = min(kEncodeBatchMax, count - i);
        const cudaError_t err =
            encode_batch<kEncodeBatchMax, false>(items + i, c, ws, status, timeout_ns, first_ticket,
                                                 stream);
        if (err != cudaSuccess) return err;
        uint64_t tiles = 0;
        for (uint32_t j = 0; j < c; ++j) tiles += encode_tiles(items[i + j].n);
        ws += (encode_workspace_bytes(tiles) + 15) & ~uint64_t(15);
    }
    return cudaSuccess;
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
