// wc_decode.cu -- fixed-length WCB1 decoder for sm_100a.
//
// Fixed-length blocks make every element's position a closed form of its
// index ("ZipServ: Fast and Memory-Efficient LLM Inference with
// Hardware-Aware Lossless Compression", Abstract: variable-length bitstreams
// break SIMT parallelism, a fixed-length format decodes in constant time per
// element, in parallel). Element i of block b sits in octet j = (i mod B)/8 at
// byte 16*offs[b] + j*w_b of the exponent plane, lane t = i mod 8 at bits
// [t*w_b, (t+1)*w_b); its mantissa byte is byte i of the mantissa plane.
//
// The kernel is persistent and warp-specialised. Each thread block walks the
// 8192-element tiles blockIdx.x, blockIdx.x + gridDim.x, ... of the batch
// through a ring of kStages shared-memory stages guarded by mbarriers:
//   producer warp   per tile: reads and checks the block headers and offsets
//                   (w <= 8, base 0 when raw, offsets equal to the prefix sum
//                   of the block sizes, every byte inside the stream), writes
//                   per-block decode constants into the stage, and issues two
//                   bulk asynchronous copies (cp.async.bulk) -- the tile's
//                   mantissa bytes and its exponent payload, both contiguous
//                   and 16-byte aligned -- that complete on the stage's
//                   "full" barrier;
//   8 consumer warps per tile: wait on "full", decode 16 elements per chunk
//                   (2 chunks per thread) from shared memory by reversing the
//                   hierarchical halving (octet -> quads -> pairs), add the
//                   base, merge sign and mantissa, write 16-byte stores, and
//                   release the stage on its "empty" barrier.
// The decoding warps never wait on global-memory latency and never meet at a
// block-wide barrier. Every mbarrier wait is bounded by the device timer; on
// expiry the kernel reports WC_ERR_TIMEOUT and returns.
//
// A batch of tensors is one launch: the per-tensor descriptors travel as
// launch parameters and the producer advances through them as its tiles do.
//
// Escape-coded streams (header flags bit 1) use the same ring; their consumer
// warps each own a 1024-element segment of the tile, so that an escaped
// element's place in its block's exception list is a warp prefix count of the
// escapes before it (segmented by block for B < 1024, carried across the
// segment's two steps for B >= 1024, and, for B > 1024, offset by the escape
// totals of the block's earlier segments, which their warps post to shared
// memory; a warp waits only for those warps).
#include <mutex>
#include <type_traits>

#include "wc_escape_core.cuh"

namespace wc {
namespace {

constexpr int kConsumerWarps = kThreads / 32;  // 8
constexpr int kProducerWarp = kConsumerWarps;
constexpr int kDecodeThreads = kThreads + 32;  // 288
constexpr int kSegment = kTile / kConsumerWarps;  // 1024: an escape consumer warp's share of a tile
// FP32 stages also hold the tile's low halves (16 KB), so they are fewer.
template <int KIND>
constexpr int stages_of() { return KIND == kKindF32 ? 3 : 4; }

template <int MAXI>
struct DecodeParams {
    int32_t* status;
    uint32_t count;
    uint32_t pad;
    uint64_t total_tiles;
    uint64_t tile_begin[MAXI + 1];  // first global tile of each item; [count] = total
    DecodeItem item[MAXI];
};

struct __align__(16) StageInfo {
    uint16_t* out;    // the tile's first output element
    uint32_t tile_n;  // elements to decode (0: nothing, e.g. a corrupt tile)
    uint32_t log2B;
};

// Per-block decode constants, computed once per block by the producer.
//   t0 = {byte offset of the block's payload in the staged bytes, w, 2w, 4w}
//   t1 = {M1 = m1 | m1 << 16, m2, m4, base * 0x00800080}, mk = 2^k - 1 (m4 = ~0 when 4w = 32)
// (escape-coded streams: see commit_tile_meta_escape)
template <int KIND>
struct __align__(16) Stage {
    uint8_t man[kTile];
    uint8_t exp[kTile + 16];
    uint16_t low[KIND == kKindF32 ? kTile : 8];  // FP32: the tile's low halves
    uint4 t0[kMaxBlocksPerTile];
    // escape-coded stages keep 8 bytes here, so that three thread blocks fit an SM
    typename std::conditional<KIND == kKindEscape, uint2, uint4>::type t1[kMaxBlocksPerTile];
    StageInfo info;
};

// Escape-coded tiles with blocks longer than a consumer warp's segment: each
// warp's escape total for the stage's tile and the tile's sequence number
// (its round-robin index + 1), posted once the total is known. A warp waits
// only for the warps of the earlier segments of its block. A slot cannot be
// overwritten before its readers are done: stage s takes a new tile only
// after all eight consumer warps released it.
struct EscSegments {
    uint32_t count[stages_of<kKindEscape>()][kConsumerWarps];
    uint32_t seq[stages_of<kKindEscape>()][kConsumerWarps];
};
struct NoEscSegments {};

template <int KIND>
struct DecodeSmem {
    static constexpr int kStages = stages_of<KIND>();
    Stage<KIND> stage[kStages];
    unsigned long long full[kStages];
    unsigned long long empty[kStages];
    typename std::conditional<KIND == kKindEscape, EscSegments, NoEscSegments>::type seg;
    int abort;
};

// ---------------------------------------------------------------------------
// producer: one warp
// ---------------------------------------------------------------------------
template <int KIND>
__device__ __forceinline__ Layout layout_of_kind(uint64_t n, uint32_t B) {
    return KIND == kKindEscape ? make_layout_escape(n, B) : make_layout(n, B, KIND == kKindF32);
}

// Copy `bytes` (a multiple of 16) from page-locked host memory, read through the
// device's mapping of it, into shared memory: 16-byte loads by the whole warp,
// four in flight per lane (2 KB per warp round trip; the grid's hundreds of
// producers keep the host link busy).
__device__ __forceinline__ void warp_copy_from_host(uint8_t* dst, const uint8_t* src,
                                                    uint32_t bytes, int lane) {
    for (uint32_t base = 0; base < bytes; base += 32u * 16u * 4u) {
        uint4 v[4];
#pragma unroll
        for (int k = 0; k < 4; ++k) {
            const uint32_t off = base + (uint32_t(k) * 32u + uint32_t(lane)) * 16u;
            if (off < bytes) v[k] = *reinterpret_cast<const uint4*>(src + off);
        }
#pragma unroll
        for (int k = 0; k < 4; ++k) {
            const uint32_t off = base + (uint32_t(k) * 32u + uint32_t(lane)) * 16u;
            if (off < bytes) *reinterpret_cast<uint4*>(dst + off) = v[k];
        }
    }
}

// HOST: the streams are in page-locked host memory; the producer reads each
// tile's bytes over the host link itself instead of issuing bulk copies, so
// the transfer and the decode of earlier tiles overlap in one launch.
template <int MAXI, int KIND, bool HOST>
__device__ void produce(const DecodeParams<MAXI>& P, DecodeSmem<KIND>& sm, int lane) {
    constexpr int kStages = DecodeSmem<KIND>::kStages;
    constexpr bool F32 = KIND == kKindF32;
    uint32_t it = 0;
    DecodeItem I = P.item[0];
    Layout L = layout_of_kind<KIND>(I.n, I.block);
    int issued_round[kStages];  // last round whose bulk copies were issued, per stage
    for (int s = 0; s < kStages; ++s) issued_round[s] = -1;
    for (uint64_t i = 0;; ++i) {
        const uint64_t t = blockIdx.x + i * gridDim.x;
        if (t >= P.total_tiles) break;
        const int s = int(i % kStages);
        const uint32_t round = uint32_t(i / kStages);
        if (round > 0 && !mbar_wait(&sm.empty[s], (round & 1u) ^ 1u, &sm.abort, 256)) {
            if (lane == 0) {
                report(P.status, kStatusTimeout);
                sm.abort = 1;
                // wait (bounded) for this warp's copies still in flight into shared memory
                for (int k = 0; k < kStages; ++k)
                    if (issued_round[k] >= 0)
                        mbar_wait(&sm.full[k], uint32_t(issued_round[k]) & 1u, nullptr);
            }
            return;
        }
        if (t >= P.tile_begin[it + 1]) {  // tiles only move forward: advance the item
            while (t >= P.tile_begin[it + 1]) ++it;
            I = P.item[it];
            L = layout_of_kind<KIND>(I.n, I.block);
        }
        const uint64_t lt = t - P.tile_begin[it];
        if (lt == 0 && lane == 0) check_container(I, L, P.status);
        Stage<KIND>& st = sm.stage[s];

        uint32_t tile_n = 0, len16 = 0, man_bytes = 0;
        uint64_t start = 0;
        bool bad = false;
        if (L.n > 0) {
            const uint64_t tile_start = lt * kTile;
            tile_n = uint32_t(min(uint64_t(kTile), L.n - tile_start));
            const TileMeta meta = load_tile_meta(I.stream, L, tile_start, tile_n, lane);
            if constexpr (KIND == kKindEscape)
                bad = !commit_tile_meta_escape(meta, I.stream, L, I.stream_bytes, tile_n, st.t0,
                                               st.t1, st.exp, start, len16, lane);
            else
                bad = !commit_tile_meta(meta, I.stream, L, I.stream_bytes, tile_n, st.t0, st.t1,
                                        st.exp, start, len16, lane);
            if (!bad) {
                man_bytes = (tile_n + 15u) & ~15u;  // inside the 128-byte padded plane
                if (lane == 0) {  // FP32 outputs are 32-bit words
                    uint16_t* out = F32 ? reinterpret_cast<uint16_t*>(
                                              reinterpret_cast<uint32_t*>(I.out) + tile_start)
                                        : I.out + tile_start;
                    st.info = StageInfo{out, tile_n, L.log2_block};
                }
            } else {
                if (lane == 0) report(P.status, kStatusCorrupt);
            }
        }
        if (L.n == 0 || bad) {
            if (lane == 0) st.info = StageInfo{nullptr, 0u, 0u};
            tile_n = 0;
        }
        __syncwarp();
        if (HOST && tile_n != 0) {
            const uint8_t* S = I.stream;
            warp_copy_from_host(st.man, S + L.off_man + lt * kTile, man_bytes, lane);
            if (len16) warp_copy_from_host(st.exp, S + L.off_exp + start, len16, lane);
            __syncwarp();  // every lane's stores precede lane 0's arrive
        }
        if (lane == 0) {
            if (tile_n == 0 || HOST) {
                mbar_arrive(&sm.full[s]);
            } else {
                const uint32_t low_bytes = F32 ? (2u * tile_n + 15u) & ~15u : 0u;
                mbar_arrive_expect_tx(&sm.full[s], man_bytes + len16 + low_bytes);
                const uint8_t* S = I.stream;
                bulk_load(st.man, S + L.off_man + lt * kTile, man_bytes, &sm.full[s]);
                if (len16) bulk_load(st.exp, S + L.off_exp + start, len16, &sm.full[s]);
                if (F32)  // inside the 128-byte padded low plane
                    bulk_load(st.low, S + L.off_low + 2 * lt * kTile, low_bytes, &sm.full[s]);
                issued_round[s] = int(round);
            }
        }
    }
}

// ---------------------------------------------------------------------------
// consumers: eight warps
// ---------------------------------------------------------------------------
// FP32 words 2k, 2k+1 from a pair of high halves and a pair of low halves.
__device__ __forceinline__ uint4 join_fp32(uint32_t hi01, uint32_t lo01, uint32_t hi23,
                                           uint32_t lo23) {
    return make_uint4(prmt(lo01, hi01, 0x5410u), prmt(lo01, hi01, 0x7632u),
                      prmt(lo23, hi23, 0x5410u), prmt(lo23, hi23, 0x7632u));
}

template <int MAXI, int KIND>
__device__ void consume(const DecodeParams<MAXI>& P, DecodeSmem<KIND>& sm, int tid, int lane) {
    constexpr int kStages = DecodeSmem<KIND>::kStages;
    constexpr bool F32 = KIND == kKindF32;
    for (uint64_t i = 0;; ++i) {
        const uint64_t t = blockIdx.x + i * gridDim.x;
        if (t >= P.total_tiles) break;
        const int s = int(i % kStages);
        const uint32_t round = uint32_t(i / kStages);
        if (!mbar_wait(&sm.full[s], round & 1u, &sm.abort)) {
            if (lane == 0) {
                report(P.status, kStatusTimeout);
                sm.abort = 1;
            }
            return;
        }
        const Stage<KIND>& st = sm.stage[s];
        const StageInfo info = st.info;
        const uint32_t bmask = (1u << info.log2B) - 1u;
#pragma unroll
        for (int k = 0; k < kChunksPerThread; ++k) {
            const uint32_t el = uint32_t(tid + k * kThreads) * kChunk;
            if (el >= info.tile_n) continue;
            const uint4 M = *reinterpret_cast<const uint4*>(st.man + el);
            const uint32_t bl = el >> info.log2B;
            const uint4 t0 = st.t0[bl], t1 = st.t1[bl];
            const uint32_t q = t0.x + ((el & bmask) >> 3) * t0.y;
            uint4 r0, r1;
            decode_chunk(st.exp, q, M, t0, t1, r0, r1);
            if (F32) {  // join each high half with its low half
                uint32_t* dst = reinterpret_cast<uint32_t*>(info.out) + el;
                const uint4 l0 = *reinterpret_cast<const uint4*>(st.low + el);
                const uint4 l1 = *reinterpret_cast<const uint4*>(st.low + el + 8);
                const uint4 y[4] = {join_fp32(r0.x, l0.x, r0.y, l0.y), join_fp32(r0.z, l0.z, r0.w, l0.w),
                                    join_fp32(r1.x, l1.x, r1.y, l1.y), join_fp32(r1.z, l1.z, r1.w, l1.w)};
                if (info.tile_n - el >= kChunk) {
#pragma unroll
                    for (int j = 0; j < 4; ++j) st_stream_v4(dst + 4 * j, y[j]);
                } else {
                    const uint32_t words[16] = {y[0].x, y[0].y, y[0].z, y[0].w, y[1].x, y[1].y,
                                                y[1].z, y[1].w, y[2].x, y[2].y, y[2].z, y[2].w,
                                                y[3].x, y[3].y, y[3].z, y[3].w};
                    const uint32_t nv = info.tile_n - el;
                    for (uint32_t e = 0; e < nv; ++e) dst[e] = words[e];
                }
            } else {
                uint16_t* dst = info.out + el;
                if (info.tile_n - el >= kChunk) {
                    st_stream_v4(dst, r0);
                    st_stream_v4(dst + 8, r1);
                } else {
                    const uint32_t words[8] = {r0.x, r0.y, r0.z, r0.w, r1.x, r1.y, r1.z, r1.w};
                    const uint32_t nv = info.tile_n - el;
                    for (uint32_t e = 0; e < nv; ++e)
                        dst[e] = uint16_t(words[e >> 1] >> (16 * (e & 1)));
                }
            }
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&sm.empty[s]);
    }
}

// ---------------------------------------------------------------------------
// consumers of escape-coded streams: eight warps, one 1024-element segment each
// ---------------------------------------------------------------------------
// One chunk of an escape-coded tile in a consumer lane's registers.
struct EscChunk {
    uint32_t el;      // first element (tile-relative)
    uint32_t q;       // staged byte of its first code
    uint32_t E[4];    // exponent bytes
    uint32_t esc[4];  // escape flags (bit 8t+7 of word j: element 4j+t)
    uint4 M;          // sign+mantissa bytes
    uint4 t0;         // its block's constants
    uint2 t1;
    uint32_t count;   // escapes in the chunk
    bool active;
};

// FULL: a full tile (every chunk active), without the tail's selects and checks.
template <bool FULL>
__device__ __forceinline__ void load_esc_meta(const Stage<kKindEscape>& st, uint32_t el,
                                              uint32_t tile_n, uint32_t log2B, EscChunk& c) {
    c.el = el;
    c.active = FULL || el < tile_n;
    c.count = 0;
    // an inactive chunk (past the end of the tile) decodes staged byte 0 as
    // width 3 and is never stored
    const uint32_t bl = c.active ? el >> log2B : 0u;
    c.t0 = c.active ? st.t0[bl] : make_uint4(0u, 3u, 0u, 0u);
    c.t1 = st.t1[bl];
    c.M = *reinterpret_cast<const uint4*>(st.man + (c.active ? el : 0u));
    c.q = c.t0.x + ((el & ((1u << log2B) - 1u)) >> 3) * c.t0.y;
    if (!c.active) c.q = 0;
}

// The last chunk of a stream: bits past the block's codes are not codes (they
// hold its exceptions and padding).
template <bool FULL>
__device__ __forceinline__ void finish_esc_codes(uint32_t tile_n, EscChunk& c) {
    const uint32_t nv = tile_n - c.el;
    if (!FULL && nv < uint32_t(kChunk)) {
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const int valid = int(nv) - 4 * j;
            if (valid < 4) c.esc[j] &= valid <= 0 ? 0u : (0xFFFFFFFFu >> (32 - 8 * valid));
        }
    }
    c.count = escape_count(c.esc);
}

// Decode the codes of a lane's chunks: 3-bit codes (the width escape-coded
// Gaussian weights take) through code specialised on the width, any other
// width through the run-time path.
// Both chunks are first decoded as 3-bit codes without a branch (so that their
// shared-memory loads can be scheduled together); a chunk of another width is
// then decoded again through the run-time path.
template <bool FULL>
__device__ __forceinline__ void decode_esc_pair(const Stage<kKindEscape>& st, uint32_t tile_n,
                                                EscChunk& c0, EscChunk& c1) {
    chunk_exponents<3>(st.exp, c0.q, c0.t1.x, c0.t1.y, c0.E, c0.esc);
    chunk_exponents<3>(st.exp, c1.q, c1.t1.x, c1.t1.y, c1.E, c1.esc);
    if (c0.t0.y != 3u) chunk_exponents_rt(st.exp, c0.q, c0.t0.y, c0.t1.x, c0.t1.y, c0.E, c0.esc);
    if (c1.t0.y != 3u) chunk_exponents_rt(st.exp, c1.q, c1.t0.y, c1.t1.x, c1.t1.y, c1.E, c1.esc);
    if (FULL || c0.active) finish_esc_codes<FULL>(tile_n, c0);
    if (FULL || c1.active) finish_esc_codes<FULL>(tile_n, c1);
}

// Put the chunk's exceptions -- staged bytes [p, p + count), in element order --
// into its escaped bytes. A word with one escape (all but a few in a thousand
// for Gaussian weights) takes its exception with a byte mask; a word with more
// goes byte by byte.
__device__ __forceinline__ void patch_esc_chunk(const uint8_t* exp, uint32_t p, EscChunk& c) {
    uint32_t k[4], multi = 0;
#pragma unroll
    for (int j = 0; j < 4; ++j) {  // without branches: a word without escapes keeps its bytes
        const uint32_t esc = c.esc[j];
        k[j] = __popc(esc);
        multi |= k[j] >> 1;
        const uint32_t mask = (esc >> 7) * 0xFFu;
        c.E[j] ^= (c.E[j] ^ (uint32_t(exp[p]) * 0x01010101u)) & mask;
        p += k[j];
    }
    if (multi) {  // some word holds two or more escapes: place its bytes one by one
#pragma unroll
        for (int j = 3; j >= 0; --j) {
            p -= k[j];
            if (k[j] > 1u) {
                uint32_t m = c.esc[j], r = p, E = c.E[j];
                do {
                    const uint32_t byte = (uint32_t(__ffs(int(m))) - 1u) >> 3;  // bit 8b + 7 -> b
                    const uint32_t sel = (0x3210u & ~(0xFu << (4 * byte))) | (4u << (4 * byte));
                    E = prmt(E, exp[r++], sel);
                    m &= m - 1u;
                } while (m);
                c.E[j] = E;
            }
        }
    }
}

// Patch the chunk's escaped elements with their exceptions (the `before`-th
// exception of its block onwards), check the block's payload size if the
// chunk holds the block's last element, and store the 16 BF16 words.
template <bool FULL>
__device__ __forceinline__ bool finish_esc_chunk(const Stage<kKindEscape>& st, EscChunk& c,
                                                 uint32_t before, uint32_t tile_n, uint32_t log2B,
                                                 uint16_t* out) {
    bool bad = false;
    if (c.count) {
        const uint32_t p = c.t0.x + c.t0.z + before;
        if (p + c.count > c.t0.w)
            bad = true;
        else
            patch_esc_chunk(st.exp, p, c);
    }
    const uint32_t next = c.el + uint32_t(kChunk);
    // (a full tile ends on a block boundary)
    if (((next & ((1u << log2B) - 1u)) == 0u || (!FULL && next >= tile_n)) &&
        ((c.t0.z + before + c.count + 15u) & ~15u) != c.t0.w - c.t0.x)
        bad = true;
    uint4 r0, r1;
    merge_quad(c.E[0], c.M.x, r0.x, r0.y);
    merge_quad(c.E[1], c.M.y, r0.z, r0.w);
    merge_quad(c.E[2], c.M.z, r1.x, r1.y);
    merge_quad(c.E[3], c.M.w, r1.z, r1.w);
    uint16_t* dst = out + c.el;
    if (FULL || tile_n - c.el >= uint32_t(kChunk)) {
        st_stream_v4(dst, r0);
        st_stream_v4(dst + 8, r1);
    } else {
        const uint32_t words[8] = {r0.x, r0.y, r0.z, r0.w, r1.x, r1.y, r1.z, r1.w};
        const uint32_t nv = tile_n - c.el;
        for (uint32_t e = 0; e < nv; ++e) dst[e] = uint16_t(words[e >> 1] >> (16 * (e & 1)));
    }
    return bad;
}

// Wait (bounded by the device timer, like every wait of the kernel) until a
// warp's posted sequence number in shared memory reaches `tag`.
__device__ __forceinline__ bool wait_tag(const uint32_t* p, uint32_t tag, volatile int* abort) {
    const volatile uint32_t* v = p;
    if (*v == tag) return true;
    const uint64_t t0 = global_timer_ns();
    while (*v != tag) {
        if (*abort || global_timer_ns() - t0 > kWaitLimitNs) return false;
    }
    return true;
}

template <int MAXI>
__device__ void consume_escape(const DecodeParams<MAXI>& P, DecodeSmem<kKindEscape>& sm, int tid,
                               int lane, int warp) {
    constexpr int kStages = DecodeSmem<kKindEscape>::kStages;
    (void)tid;
    for (uint64_t i = 0;; ++i) {
        const uint64_t t = blockIdx.x + i * gridDim.x;
        if (t >= P.total_tiles) break;
        const int s = int(i % kStages);
        const uint32_t round = uint32_t(i / kStages);
        if (!mbar_wait(&sm.full[s], round & 1u, &sm.abort)) {
            if (lane == 0) {
                report(P.status, kStatusTimeout);
                sm.abort = 1;
            }
            return;
        }
        const Stage<kKindEscape>& st = sm.stage[s];
        const StageInfo info = st.info;
        const uint32_t log2B = info.log2B, B = 1u << log2B;
        const uint32_t seg = uint32_t(warp) * kSegment;
        bool bad = false;
        const bool active = seg < info.tile_n;  // the same for the whole warp
        const bool full = info.tile_n == uint32_t(kTile);
        // both 512-element steps of the segment at once: chunk k of this lane
        // starts at seg + 512k + 16 lane
        EscChunk c0, c1;
        uint32_t incl = 0, v = 0;
        if (active) {
            if (full) {
                load_esc_meta<true>(st, seg + 16u * uint32_t(lane), kTile, log2B, c0);
                load_esc_meta<true>(st, seg + 512u + 16u * uint32_t(lane), kTile, log2B, c1);
                decode_esc_pair<true>(st, kTile, c0, c1);
            } else {
                load_esc_meta<false>(st, seg + 16u * uint32_t(lane), info.tile_n, log2B, c0);
                load_esc_meta<false>(st, seg + 512u + 16u * uint32_t(lane), info.tile_n, log2B, c1);
                decode_esc_pair<false>(st, info.tile_n, c0, c1);
            }
            // one prefix count for both steps (step k's counts in bits [16k, 16k + 16)),
            // segmented by block: B/16 lanes hold one block of a step when B < 512
            v = c0.count | (c1.count << 16);
            incl = v;
            if (B >= 512u) {
#pragma unroll
                for (int d = 1; d < 32; d <<= 1) {
                    const uint32_t y = __shfl_up_sync(0xFFFFFFFFu, incl, d);
                    if (lane >= d) incl += y;
                }
            } else {
                const uint32_t group = B >> 4;
                for (uint32_t d = 1; d < group; d <<= 1) {
                    const uint32_t y = __shfl_up_sync(0xFFFFFFFFu, incl, d, int(group));
                    if ((uint32_t(lane) & (group - 1u)) >= d) incl += y;
                }
            }
        }
        // Blocks longer than a segment: the escapes of the block's earlier
        // segments, from the totals their warps post.
        const uint32_t last = B >= uint32_t(kSegment) ? __shfl_sync(0xFFFFFFFFu, incl, 31) : 0u;
        uint32_t carry = 0;
        if (B > uint32_t(kSegment)) {
            const uint32_t tag = uint32_t(i) + 1u;
            if (lane == 0) {
                sm.seg.count[s][warp] = (last & 0xFFFFu) + (last >> 16);
                __threadfence_block();
                *reinterpret_cast<volatile uint32_t*>(&sm.seg.seq[s][warp]) = tag;
            }
            // lane k waits for the warp of the block's k-th segment, if earlier
            const uint32_t w0 = (seg & ~(B - 1u)) / uint32_t(kSegment);
            const uint32_t wk = w0 + uint32_t(lane);
            uint32_t c = 0;
            bool ok = true;
            if (wk < uint32_t(warp)) {
                ok = wait_tag(&sm.seg.seq[s][wk], tag, &sm.abort);
                __threadfence_block();
                c = sm.seg.count[s][wk];
            }
            if (!__all_sync(0xFFFFFFFFu, ok)) {
                if (lane == 0) {
                    report(P.status, kStatusTimeout);
                    sm.abort = 1;
                }
                return;
            }
            carry = __reduce_add_sync(0xFFFFFFFFu, c);
        }
        if (active) {
            const uint32_t excl = incl - v;
            uint32_t before0 = excl & 0xFFFFu, before1 = excl >> 16;
            if (B >= uint32_t(kSegment)) {  // step 1 continues step 0's block
                before0 += carry;
                before1 += carry + (last & 0xFFFFu);
            }
            if (full) {
                bad |= finish_esc_chunk<true>(st, c0, before0, kTile, log2B, info.out);
                bad |= finish_esc_chunk<true>(st, c1, before1, kTile, log2B, info.out);
            } else {
                if (c0.active) bad |= finish_esc_chunk<false>(st, c0, before0, info.tile_n, log2B, info.out);
                if (c1.active) bad |= finish_esc_chunk<false>(st, c1, before1, info.tile_n, log2B, info.out);
            }
        }
        if (__any_sync(0xFFFFFFFFu, bad) && lane == 0) report(P.status, kStatusCorrupt);
        __syncwarp();
        if (lane == 0) mbar_arrive(&sm.empty[s]);
    }
}

template <int MAXI, int KIND, bool HOST>
__global__ void __launch_bounds__(kDecodeThreads)
    decode_kernel(const __grid_constant__ DecodeParams<MAXI> P) {
    constexpr int kStages = DecodeSmem<KIND>::kStages;
    extern __shared__ __align__(128) unsigned char smem_raw[];
    DecodeSmem<KIND>& sm = *reinterpret_cast<DecodeSmem<KIND>*>(smem_raw);
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    if (tid == 0) {
        for (int s = 0; s < kStages; ++s) {
            mbar_init(&sm.full[s], 1);                // the producer's arrive (+ copied bytes)
            mbar_init(&sm.empty[s], kConsumerWarps);  // one arrive per consumer warp
        }
        if constexpr (KIND == kKindEscape)
            for (int s = 0; s < kStages; ++s)
                for (int w = 0; w < kConsumerWarps; ++w) sm.seg.seq[s][w] = 0;
        sm.abort = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    __syncthreads();
    if (warp == kProducerWarp)
        produce<MAXI, KIND, HOST>(P, sm, lane);
    else if constexpr (KIND == kKindEscape)
        consume_escape<MAXI>(P, sm, tid, lane, warp);
    else
        consume<MAXI, KIND>(P, sm, tid, lane);
}

// Persistent grid: as many resident thread blocks as the SMs hold, never more
// than there are tiles. Computed once per device and kernel instantiation.
template <int MAXI, int KIND, bool HOST>
cudaError_t grid_for(uint64_t tiles, unsigned* grid) {
    static std::mutex mu;
    static int per_device[64];  // 0 = not yet known
    int dev = 0;
    cudaError_t err = cudaGetDevice(&dev);
    if (err != cudaSuccess) return err;
    if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
    std::lock_guard<std::mutex> lock(mu);
    if (per_device[dev] == 0) {
        err = cudaFuncSetAttribute(decode_kernel<MAXI, KIND, HOST>,
                                   cudaFuncAttributeMaxDynamicSharedMemorySize,
                                   int(sizeof(DecodeSmem<KIND>)));
        if (err != cudaSuccess) return err;
        int sms = 0, per_sm = 0;
        err = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
        if (err != cudaSuccess) return err;
        err = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, decode_kernel<MAXI, KIND, HOST>,
                                                            kDecodeThreads, sizeof(DecodeSmem<KIND>));
        if (err != cudaSuccess) return err;
        per_device[dev] = (per_sm > 0 ? per_sm : 1) * sms;
    }
    const uint64_t cap = uint64_t(per_device[dev]);
    *grid = unsigned(tiles < cap ? tiles : cap);
    return cudaSuccess;
}

template <int MAXI, int KIND, bool HOST>
cudaError_t launch_batch(const DecodeItem* items, uint32_t count, int32_t* status,
                         cudaStream_t stream) {
    static_assert(sizeof(DecodeParams<MAXI>) <= 32000, "launch parameters exceed the limit");
    DecodeParams<MAXI> p;
    p.status = status;
    p.count = count;
    p.pad = 0;
    uint64_t tiles = 0;
    for (uint32_t i = 0; i < count; ++i) {
        p.tile_begin[i] = tiles;
        p.item[i] = items[i];
        const uint64_t nt = num_tiles(items[i].n);
        tiles += nt ? nt : 1;  // an empty tensor still gets one tile to check its header
    }
    p.tile_begin[count] = tiles;
    p.total_tiles = tiles;
    if (tiles == 0) return cudaSuccess;
    unsigned grid = 0;
    cudaError_t err = grid_for<MAXI, KIND, HOST>(tiles, &grid);
    if (err != cudaSuccess) return err;
    decode_kernel<MAXI, KIND, HOST><<<grid, kDecodeThreads, sizeof(DecodeSmem<KIND>), stream>>>(p);
    return cudaGetLastError();
}

}  // namespace

constexpr uint32_t kBatchMax = 512;

template <int KIND, bool HOST>
cudaError_t launch_kind(const DecodeItem* items, uint32_t count, int32_t* status,
                        cudaStream_t stream) {
    if (count == 1) return launch_batch<1, KIND, HOST>(items, 1, status, stream);
    for (uint32_t i = 0; i < count; i += kBatchMax) {
        const uint32_t c = min(kBatchMax, count - i);
        const cudaError_t err = launch_batch<kBatchMax, KIND, HOST>(items + i, c, status, stream);
        if (err != cudaSuccess) return err;
    }
    return cudaSuccess;
}

cudaError_t launch_decode(const DecodeItem* items, uint32_t count, int32_t* status,
                          cudaStream_t stream, int kind, bool host_streams) {
    if (kind == kKindF32) {  // FP32 streams: one tensor per call, device streams only
        if (host_streams) return cudaErrorInvalidValue;
        for (uint32_t i = 0; i < count; ++i) {
            const cudaError_t err = launch_batch<1, kKindF32, false>(items + i, 1, status, stream);
            if (err != cudaSuccess) return err;
        }
        return cudaSuccess;
    }
    if (kind == kKindEscape)
        return host_streams ? launch_kind<kKindEscape, true>(items, count, status, stream)
                            : launch_kind<kKindEscape, false>(items, count, status, stream);
    return host_streams ? launch_kind<kKindPlain, true>(items, count, status, stream)
                        : launch_kind<kKindPlain, false>(items, count, status, stream);
}

}  // namespace wc
