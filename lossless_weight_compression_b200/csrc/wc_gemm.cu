// wc_gemm.cu -- fused decompression and matrix products on the sm_100a tensor cores.
//
// Y[t][r] = sum_c W[r][c] * X[t][c] for t < tokens (1..128), where the BF16
// weight matrix W (rows x cols, row-major) is held only as a WCB1 stream: each
// 128 x 128 slice of W is decoded on chip and fed to the tensor cores from
// tensor memory, so decoded weights never touch HBM ("ZipServ: Fast and
// Memory-Efficient LLM Inference with Hardware-Aware Lossless Compression",
// Abstract: decompression fused into the matrix product, load compressed and
// compute decompressed).
//
// One thread block per SM, persistent. A unit is 128 consecutive rows of one
// matrix (the MMA's M) times all tokens (its N, padded to a multiple of 16),
// swept over cols in slices of 128. Each slice passes through a chain of
// roles joined by mbarrier rings, so that no role waits for all the others
// at once:
//   - one thread starts the slice's mantissa bytes (one 2-D TMA load,
//     128-byte swizzled) and another its activations (two 2-D TMA loads);
//   - four row warps, one lane per row and a few slices ahead, check each
//     row's block header and offset and fetch the row's exponent bytes (a
//     128-column slice of a row is 16 whole octets of one block, 16*w
//     contiguous bytes; 16-byte cp.async pieces);
//   - eight transcoding warps unpack those bits into one exponent byte per
//     weight (base + v), eight lanes per row; a step of four rows whose widths
//     are all 4 takes a nibble path (escape-coded streams: also a width-3
//     path), any other step a path for every width; escape-coded streams
//     (header flags bit 1) also have their escapes ranked and replaced by the
//     block's exception bytes here;
//   - eight writing warps, one lane per row (a warp's lanes are the 32 tensor
//     memory lanes its rank in the warpgroup may access), merge each exponent
//     byte with its sign+mantissa byte into BF16 and store the slice's A
//     operand into tensor memory with tcgen05.st: the same few instructions
//     for every width;
//   - one thread issues tcgen05.mma (A from tensor memory, activations from
//     shared memory; BF16 x BF16 -> FP32, M = 128, K = 16), spreading
//     consecutive MMAs over several accumulators in tensor memory;
//   - four epilogue warps sum a finished unit's accumulators (tcgen05.ld) in a
//     fixed order and write Y while the next unit accumulates.
// Every wait is bounded by the device timer, after which the block stops and
// reports WC_ERR_TIMEOUT. Each unit sums its row in the same order on every
// run, so Y is reproducible bit for bit.
#include <cuda.h>
#include <cudaTypedefs.h>

#include <string.h>

#include <algorithm>
#include <mutex>

#include "wc_escape_core.cuh"

namespace wc {
namespace {

constexpr uint32_t kTileRows = 128;    // MMA M
constexpr uint32_t kSliceCols = 128;   // columns per pipeline slice (8 MMAs of K = 16)
constexpr uint32_t kExpPitch = 144;    // bytes per row of a staged slice (<= 128 used, +16 spreads banks)
constexpr uint32_t kManStage = kTileRows * kSliceCols;      // 16 KB: sign+mantissa bytes
constexpr uint32_t kRawStage = kTileRows * kExpPitch;       // 18 KB: packed exponent bits
constexpr uint32_t kMetaStage = kTileRows * 4;              // w | base << 8 | flags << 16 per row
// escape-coded streams: per row and stage, the first kExcBytes bytes of the
// row's block's exception list, and {list length, list address} of the block
constexpr uint32_t kExcBytes = 48;
constexpr uint32_t kExcStage = kTileRows * kExcBytes;       // 6 KB
constexpr uint32_t kEMetaStage = kTileRows * 16;            // 2 KB
constexpr uint32_t kMetaFirst = 1u << 16;  // the slice starts the row's block
constexpr uint32_t kMetaLast = 1u << 17;   // the slice ends the row's block
constexpr uint32_t kEStage = kTileRows * kExpPitch;         // 18 KB: exponent bytes
constexpr uint32_t kMaxRing = 4;     // mantissa and packed-exponent rings: 3 or 4 stages
constexpr uint32_t kERing = 2;       // exponent-byte ring
constexpr uint32_t kARing = 4;       // A operand stages in tensor memory
constexpr uint32_t kMaxXRing = 8;    // activation stages: as many as fit, up to 8
constexpr uint32_t kACol0 = 256;     // tensor memory column of A stage 0 (accumulators below)
constexpr uint32_t kACols = kSliceCols / 2;  // 64 columns: 128 BF16 per lane
constexpr uint32_t kSmemLimit = 232448;                     // 227 KB per block

constexpr int kProducerWarp = 0;
constexpr int kMmaWarp = 1;
constexpr int kXWarp = 2;        // warp 3 has no role
constexpr int kEpiWarp0 = 4;     // 4..7: warp % 4 is the tensor memory lane quarter
constexpr int kEpiWarps = 4;
constexpr int kWrtWarp0 = 8;     // 8..15: lane quarter warp % 4, column half (warp - 8) / 4
constexpr int kWrtWarps = 8;
constexpr int kTrWarp0 = 16;     // 16..23: 16 rows each
constexpr int kTrWarps = 8;
constexpr int kRowWarp0 = 24;    // 24..27: one lane per row of the tile
constexpr int kRowWarps = 4;
constexpr int kGemmThreads = 32 * (kRowWarp0 + kRowWarps);  // 896
static_assert(kWrtWarp0 % 4 == 0 && kEpiWarp0 % 4 == 0, "lane quarters follow the warp rank");
static_assert(kTrWarps * 16 == int(kTileRows), "each transcoding warp owns 16 rows");
static_assert(kACol0 + kARing * kACols <= 512, "tensor memory holds 512 columns");

template <int MAXI>
struct GemmParams {
    CUtensorMap man_map[MAXI];   // mantissa plane as a (rows x cols) u8 tensor
    CUtensorMap x_map[MAXI];     // activations as a (tokens x cols) BF16 tensor
    GemvItem item[MAXI];
    uint64_t unit_begin[MAXI + 1];
    int32_t* status;
    uint64_t total_units;
    uint32_t count;
    uint32_t tokens;      // valid rows of X and Y
    uint32_t nt;          // tokens rounded up to a multiple of 16: the MMA's N
    uint32_t ring;        // stages of the mantissa and packed-exponent rings (3 or 4)
    uint32_t xring;       // activation stages (2..8)
    uint32_t nacc;        // accumulators per unit (1, 2 or 4): MMA k goes to accumulator k % nacc
    uint32_t nbuf;        // units in flight in tensor memory (1 or 2)
    uint32_t escape;      // 1: escape-coded streams (cols a multiple of the block size)
    uint32_t pad[2];
};

// Shared memory, carved at run time (sizes depend on nt and the ring depth).
// The swizzled regions start 1024-byte aligned, as the 128-byte swizzle
// pattern repeats every 8 rows of 128 bytes and is a function of the address.
struct GemmCtl {
    unsigned long long man_full[kMaxRing], man_empty[kMaxRing];
    unsigned long long raw_full[kMaxRing], raw_empty[kMaxRing];
    unsigned long long e_full[kERing], e_empty[kERing];
    unsigned long long a_full[kARing], a_empty[kARing];
    unsigned long long x_full[kMaxXRing], x_empty[kMaxXRing];
    unsigned long long acc_full[2], acc_empty[2];
    unsigned long long drain;
    uint32_t tmem_base;
    int abort;
};

struct GemmSmem {
    GemmCtl* ctl;
    uint8_t* x;      // xring stages of nt * 256 bytes
    uint8_t* man;    // ring stages of kManStage
    uint8_t* raw;    // ring stages of kRawStage
    uint32_t* meta;  // ring stages of 128 words: w | base << 8 | flags << 16 of each row
    uint8_t* e;      // kERing stages of kEStage
    uint8_t* exc;    // escape-coded streams: ring stages of kExcStage
    uint4* emeta;    // escape-coded streams: ring stages of 128 x {length, address, 0}
};

__host__ __device__ inline uint32_t gemm_stage_bytes(bool escape) {
    return kManStage + kRawStage + kMetaStage + (escape ? kExcStage + kEMetaStage : 0u);
}

__host__ __device__ inline uint32_t gemm_smem_bytes(uint32_t nt, uint32_t ring, uint32_t xring,
                                                    bool escape) {
    return 1024 + 1024 /* control */ + xring * nt * 256 + ring * gemm_stage_bytes(escape) +
           kERing * kEStage;
}

// Ring depths for N = nt: the activation ring as deep as shared memory allows
// (up to 8: the activations of slice g can only be loaded once the MMAs of
// slice g - xring are done, so a shallow ring puts an L2 round trip on every
// few slices' critical path), then a fourth mantissa stage if it still fits.
inline void gemm_rings(uint32_t nt, bool escape, uint32_t* ring, uint32_t* xring) {
    // three mantissa stages, two when even two activation stages do not fit
    // beside three (128 tokens on escape-coded streams)
    *ring = gemm_smem_bytes(nt, 3, 2, escape) <= kSmemLimit ? 3u : 2u;
    *xring = kMaxXRing;
    while (*xring > 2 && gemm_smem_bytes(nt, *ring, *xring, escape) > kSmemLimit) --*xring;
    if (*xring == kMaxXRing && gemm_smem_bytes(nt, 4, *xring, escape) <= kSmemLimit) *ring = 4;
}

// ---------------------------------------------------------------------------
// tcgen05 / TMA helpers (PTX)
// ---------------------------------------------------------------------------
// Shared-memory matrix descriptor of a K-major operand in the 128-byte swizzled
// layout: rows of 128 bytes (64 BF16 along K), 8-row groups 1024 bytes apart
// (the stride byte offset); the leading byte offset is unused for this layout
// and set to 1; bits 46-47 hold the descriptor version (1), bits 61-63 the
// layout (2 = 128-byte swizzle).
__device__ __forceinline__ uint64_t sw128_desc(uint32_t saddr) {
    return uint64_t((saddr & 0x3FFFFu) >> 4) | (uint64_t(1) << 16) | (uint64_t(1024 >> 4) << 32) |
           (uint64_t(1) << 46) | (uint64_t(2) << 61);
}

// Instruction descriptor of kind::f16: FP32 accumulator (bits 4-5 = 1), A and
// B BF16 (bits 7-9 = 1, bits 10-12 = 1), both K-major (bits 15, 16 = 0),
// N >> 3 in bits 17-22, M >> 4 in bits 24-28.
__host__ __device__ inline uint32_t bf16_idesc(uint32_t m, uint32_t n) {
    return (1u << 4) | (1u << 7) | (1u << 10) | ((n >> 3) << 17) | ((m >> 4) << 24);
}

// D (tensor memory) [+]= A (tensor memory: row m in lane m, K pairs along the
// columns) * B (shared memory descriptor).
__device__ __forceinline__ void umma_bf16_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t bdesc,
                                             uint32_t idesc, uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d_tmem),
        "r"(a_tmem), "l"(bdesc), "r"(idesc), "r"(accumulate)
        : "memory");
}

// Arrive on `bar` once every tcgen05.mma this thread issued so far has completed.
__device__ __forceinline__ void umma_commit(unsigned long long* bar) {
    asm volatile(
        "tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
            smem_addr(bar))
        : "memory");
}

__device__ __forceinline__ void tc_fence_before() {
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}

// 16 consecutive FP32 columns of this thread's TMEM lane.
__device__ __forceinline__ void tmem_ld16(uint32_t taddr, uint32_t (&v)[16]) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,"
        "%14,%15}, [%16];"
        : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3]), "=r"(v[4]), "=r"(v[5]), "=r"(v[6]),
          "=r"(v[7]), "=r"(v[8]), "=r"(v[9]), "=r"(v[10]), "=r"(v[11]), "=r"(v[12]), "=r"(v[13]),
          "=r"(v[14]), "=r"(v[15])
        : "r"(taddr));
    asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}

// 16 consecutive 32-bit columns of this thread's TMEM lane from registers
// (asynchronous: tmem_wait_st orders them before a later hand-off).
__device__ __forceinline__ void tmem_st16(uint32_t taddr, const uint32_t (&v)[16]) {
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,"
        "%13,%14,%15,%16};" ::"r"(taddr),
        "r"(v[0]), "r"(v[1]), "r"(v[2]), "r"(v[3]), "r"(v[4]), "r"(v[5]), "r"(v[6]), "r"(v[7]),
        "r"(v[8]), "r"(v[9]), "r"(v[10]), "r"(v[11]), "r"(v[12]), "r"(v[13]), "r"(v[14]),
        "r"(v[15])
        : "memory");
}

__device__ __forceinline__ void tmem_wait_st() {
    asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
}

// 2-D tiled TMA load of the box at (c0, c1) into this block's shared memory, completing on `bar`.
__device__ __forceinline__ void tma_load_2d(void* dst, const CUtensorMap* map, int32_t c0,
                                            int32_t c1, unsigned long long* bar) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], "
        "[%1, {%2, %3}], [%4];" ::"r"(smem_addr(dst)),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(c0), "r"(c1), "r"(smem_addr(bar))
        : "memory");
}

// The mbarrier's current phase also waits for every cp.async this thread has
// started so far (no net arrival: the thread still arrives itself).
__device__ __forceinline__ void cp_async_mbar_arrive(unsigned long long* bar) {
    asm volatile("cp.async.mbarrier.arrive.shared::cta.b64 [%0];" ::"r"(smem_addr(bar)) : "memory");
}

// 16-byte asynchronous copy global -> shared through L2 (not L1).
__device__ __forceinline__ void cp_async16(uint32_t dst, const void* src) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(dst), "l"(src) : "memory");
}

__device__ __forceinline__ uint4 lds128(uint32_t saddr) {
    uint4 v;
    asm volatile("ld.shared.v4.u32 {%0,%1,%2,%3}, [%4];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                 : "r"(saddr));
    return v;
}

__device__ __forceinline__ void sts128(uint32_t saddr, uint32_t a, uint32_t b, uint32_t c,
                                       uint32_t d) {
    asm volatile("st.shared.v4.u32 [%0], {%1, %2, %3, %4};" ::"r"(saddr), "r"(a), "r"(b), "r"(c),
                 "r"(d)
                 : "memory");
}

__device__ __forceinline__ void sts64(uint32_t saddr, uint32_t a, uint32_t b) {
    asm volatile("st.shared.v2.u32 [%0], {%1,%2};" ::"r"(saddr), "r"(a), "r"(b) : "memory");
}

__device__ __forceinline__ void sts8(uint32_t saddr, uint32_t v) {
    asm volatile("st.shared.u8 [%0], %1;" ::"r"(saddr), "r"(v) : "memory");
}

template <int MAXI>
__device__ __forceinline__ uint32_t find_item(const GemmParams<MAXI>& P, uint64_t u, uint32_t from) {
    while (u >= P.unit_begin[from + 1]) ++from;
    return from;
}

__device__ __forceinline__ bool gemm_wait(unsigned long long* bar, uint32_t parity, GemmCtl& c,
                                          int32_t* status, uint32_t max_sleep_ns = 0) {
    if (mbar_wait(bar, parity, &c.abort, max_sleep_ns)) return true;
    if (!c.abort) report(status, kStatusTimeout);
    c.abort = 1;
    return false;
}

// The same wait by every lane of a warp; if any lane gives up, all do, so the
// warp stays converged for its shuffles and warp-wide tcgen05 instructions.
__device__ __forceinline__ bool gemm_wait_warp(unsigned long long* bar, uint32_t parity,
                                               GemmCtl& c, int32_t* status,
                                               uint32_t max_sleep_ns = 0) {
    const bool ok = gemm_wait(bar, parity, c, status, max_sleep_ns);
    return __all_sync(0xFFFFFFFFu, ok);
}

// ---------------------------------------------------------------------------
// The units a block works on, in rounds of gridDim.x: round k takes unit
// k*G + b when k is even and k*G + G-1-b when k is odd (b = blockIdx.x,
// G = gridDim.x), a snake over the blocks. The host numbers a batch's units
// longest first, so a block that took one of the long units of a round takes
// one of the short units of the next. Every role walks the same sequence; only
// the last round can be partial, so the first unit past the end ends the walk.
// ---------------------------------------------------------------------------
struct UnitWalk {
    uint64_t u;
    uint32_t odd;  // round parity
    __device__ __forceinline__ void start() {
        u = blockIdx.x;
        odd = 0;
    }
    __device__ __forceinline__ void next() {
        u += odd ? 1u + 2u * blockIdx.x : 2u * gridDim.x - 1u - 2u * blockIdx.x;
        odd ^= 1u;
    }
};

// the sequence of slices a block works on: its units, each swept over cols in
// slices of 128 (the producer and the activation loader walk it)
struct Cursor {
    UnitWalk w;
    uint32_t it, s, slices, row0;
    bool valid;
};

template <int MAXI>
__device__ __forceinline__ Cursor cursor_at(const GemmParams<MAXI>& P, UnitWalk w, uint32_t from) {
    Cursor c = {};
    c.w = w;
    c.valid = w.u < P.total_units;
    if (c.valid) {
        c.it = find_item(P, w.u, from);
        c.slices = P.item[c.it].cols / kSliceCols;
        c.row0 = uint32_t(w.u - P.unit_begin[c.it]) * kTileRows;
    }
    return c;
}

template <int MAXI>
__device__ __forceinline__ Cursor cursor_first(const GemmParams<MAXI>& P) {
    UnitWalk w;
    w.start();
    return cursor_at(P, w, 0);
}

template <int MAXI>
__device__ __forceinline__ Cursor cursor_next(const GemmParams<MAXI>& P, const Cursor& c) {
    if (c.s + 1 < c.slices) {
        Cursor n = c;
        ++n.s;
        return n;
    }
    UnitWalk w = c.w;
    w.next();
    return cursor_at(P, w, c.it);
}

// ---------------------------------------------------------------------------
// producer (one thread): the mantissa bytes of every slice, one 2-D TMA load
// into a free stage of the mantissa ring; and the container header of each
// matrix, once.
// ---------------------------------------------------------------------------
template <int MAXI>
__device__ void gemm_produce(const GemmParams<MAXI>& P, const GemmSmem& S) {
    GemmCtl& c = *S.ctl;
    const uint32_t R = P.ring;
    int issued[kMaxRing] = {-1, -1, -1, -1};  // to drain if the block stops early
    bool ok = true;
    uint32_t rs = 0, round = 0;  // slice g goes to stage rs = g % R in round g / R
    for (Cursor cur = cursor_first(P); cur.valid;
         cur = cursor_next(P, cur), rs = rs + 1 == R ? (++round, 0u) : rs + 1) {
        const GemvItem& I = P.item[cur.it];
        if (cur.row0 == 0 && cur.s == 0) {
            DecodeItem d;
            d.stream = I.stream;
            d.stream_bytes = I.stream_bytes;
            const uint64_t n = uint64_t(I.rows) * I.cols;
            check_container(d, P.escape ? make_layout_escape(n, I.block) : make_layout(n, I.block),
                            P.status);
        }
        if (round > 0 && !gemm_wait(&c.man_empty[rs], (round - 1) & 1u, c, P.status, 256)) {
            ok = false;
            break;
        }
        mbar_arrive_expect_tx(&c.man_full[rs], kManStage);
        tma_load_2d(S.man + rs * kManStage, &P.man_map[cur.it], int32_t(cur.s * kSliceCols),
                    int32_t(cur.row0), &c.man_full[rs]);
        issued[rs] = int(round);
    }
    // Stopped early: let the copies already started land before the block exits.
    if (!ok)
        for (uint32_t k = 0; k < R; ++k)
            if (issued[k] >= 0) mbar_wait(&c.man_full[k], uint32_t(issued[k]) & 1u, nullptr);
}

// ---------------------------------------------------------------------------
// activation loader (one thread): X for slice g goes into stage g % xring once
// the MMAs of slice g - xring have finished reading it
// ---------------------------------------------------------------------------
template <int MAXI>
__device__ void gemm_load_x(const GemmParams<MAXI>& P, const GemmSmem& S) {
    GemmCtl& c = *S.ctl;
    const uint32_t XR = P.xring;
    int x_issued[kMaxXRing];
    for (uint32_t k = 0; k < kMaxXRing; ++k) x_issued[k] = -1;
    bool ok = true;
    uint32_t xs = 0, round = 0;  // slice g: stage g % XR in round g / XR
    for (Cursor cur = cursor_first(P); cur.valid;
         cur = cursor_next(P, cur), xs = xs + 1 == XR ? (++round, 0u) : xs + 1) {
        if (round > 0 && !gemm_wait(&c.x_empty[xs], (round - 1) & 1u, c, P.status, 256)) {
            ok = false;
            break;
        }
        const int32_t k0 = int32_t(cur.s * kSliceCols);
        uint8_t* xd = S.x + xs * P.nt * 256;
        mbar_arrive_expect_tx(&c.x_full[xs], P.nt * 256);
        tma_load_2d(xd, &P.x_map[cur.it], k0, 0, &c.x_full[xs]);
        tma_load_2d(xd + P.nt * 128, &P.x_map[cur.it], k0 + 64, 0, &c.x_full[xs]);
        x_issued[xs] = int(round);
    }
    if (!ok)
        for (uint32_t k = 0; k < XR; ++k)
            if (x_issued[k] >= 0) mbar_wait(&c.x_full[k], uint32_t(x_issued[k]) & 1u, nullptr);
}

// ---------------------------------------------------------------------------
// row, transcoding and writing warps. A slice is 128 rows x 128 columns.
//
// Four row warps run a few slices ahead, one lane per row: a lane checks its
// row's block header and offset when the row enters a block (the header was
// loaded when the row entered the previous block), writes the row's width and
// base to the slice's stage, and fetches the row's 16*w exponent bytes
// (16-byte cp.async pieces). An mbarrier per stage hands the staged bytes
// over; it completes once every row's lane has arrived and all their copies
// have landed.
//
// Eight transcoding warps own 16 rows each and turn the packed bits into one
// exponent byte per weight; eight writing warps merge those with the
// sign+mantissa bytes into BF16 and store them into tensor memory.
// ---------------------------------------------------------------------------
// State of one row for the slice being prepared: where its exponent bytes
// start, how many of its block's elements are left from there, the block's
// width and base, and the header of the row's next block (loaded
// when the row enters a block, so it is in registers by the time the row gets
// there). Everything but the byte pointer and the count changes only when the
// row enters a block: once every block / 128 slices.
struct RowState {
    uint64_t b;          // the row's current block
    const uint8_t* src;  // the slice's exponent bytes
    uint32_t left;       // elements from the slice's first column to the block's end
    uint32_t w, base;
    uint32_t nh, noff;   // next block: header and offset (16-byte units)
    uint64_t nnx;        // next block: the following block's payload start
    const uint8_t* exc;  // escape-coded: the block's exception list
    uint32_t exc_len;    // escape-coded: its length with the payload's zero padding
    bool first;          // the slice is the first of the row's block
    bool valid;
};

__device__ __forceinline__ void set_width(RowState& R, uint32_t w, uint32_t base) {
    R.w = w;
    R.base = base;
}

// Unit-level constants of the slice being prepared.
struct UnitState {
    const uint8_t* stream;
    uint64_t stream_bytes, n, nb, off_exp, off_man;
    const uint16_t* hdr;
    const uint32_t* offs;
    uint32_t cols, rows, block, log2B;
};

template <int MAXI>
__device__ __forceinline__ UnitState unit_state(const GemmParams<MAXI>& P, uint32_t it) {
    const GemvItem& I = P.item[it];
    UnitState U;
    U.stream = I.stream;
    U.stream_bytes = I.stream_bytes;
    U.cols = I.cols;
    U.rows = I.rows;
    U.block = I.block;
    const Layout L = make_layout(uint64_t(I.rows) * I.cols, I.block);
    U.n = L.n;
    U.nb = L.nb;
    U.off_exp = L.off_exp;
    U.off_man = L.off_man;
    U.log2B = L.log2_block;
    U.hdr = reinterpret_cast<const uint16_t*>(I.stream + L.off_hdr);
    U.offs = reinterpret_cast<const uint32_t*>(I.stream + L.off_offs);
    return U;
}

// Start the loads of block b's header, offset and chain end (payload start of
// block b + 1, or E for the last block).
__device__ __forceinline__ void load_block(const UnitState& U, uint64_t b, uint32_t& h,
                                           uint32_t& off, uint64_t& nx) {
    h = U.hdr[b];
    off = U.offs[b];
    nx = b + 1 < U.nb ? 16ull * U.offs[b + 1] : ld_u64(U.stream + 64);
}

// The row enters the block holding element el (its header in h/off/nx; el is
// a slice's first column): set the width and base, the slice's exponent
// bytes and the block's remaining elements, checking the header, that
// the block's payload lies inside the stream (so no slice of it reads past the
// end) and, at the block's first element, the offset chain; then start loading
// the row's next block. False if corrupt (the row then decodes as w = 0).
// ESC: an escape-coded block (rows are whole blocks, so el is the block's
// first element): its payload is the codes, the exception list and zero
// padding to 16 bytes, so the offset chain bounds the list's length.
template <bool ESC>
__device__ __forceinline__ bool enter_block(const UnitState& U, RowState& R, uint64_t row,
                                            uint64_t el, uint32_t h, uint32_t off, uint64_t nx) {
    const uint64_t b = el >> U.log2B;
    const uint32_t ob = uint32_t(el) & (U.block - 1u);  // the slice's offset in the block
    const uint64_t len = min(uint64_t(U.block), U.n - (b << U.log2B));
    uint32_t w = h >> 8, base = h & 0xFFu;
    bool bad = w > 8u || (w == 8u && base != 0u);
    const uint64_t sb = 16ull * off, end = sb + ((len + 7) >> 3) * min(w, 8u);
    if (ESC) {
        const uint32_t m = (1u << min(w, 8u)) - 1u;
        bad |= ob != 0u || (w >= 1u && w <= 7u && base > 255u - m);
        bad |= nx < end || nx - sb > ((end - sb + len + 15) & ~uint64_t(15));
        bad |= (w == 0u || w == 8u) && nx - sb != ((end - sb + 15) & ~uint64_t(15));
        bad |= U.off_exp + nx > U.stream_bytes;
        R.exc = U.stream + U.off_exp + end;
        R.exc_len = bad ? 0u : uint32_t(nx - end);
    } else {
        if (ob == 0) bad |= end != nx;
        bad |= U.off_exp + end > U.stream_bytes;
    }
    if (bad) w = base = 0;
    R.b = b;
    R.left = uint32_t(len) - ob;
    R.src = U.stream + U.off_exp + sb + (ob >> 3) * w;
    R.first = true;
    set_width(R, w, base);
    // the row continues into block b + 1 inside this unit's columns?
    if (((b + 1) << U.log2B) < (row + 1) * uint64_t(U.cols)) load_block(U, b + 1, R.nh, R.noff, R.nnx);
    return !bad;
}

// Row warps: lane l of row warp p owns row 32p + l of every slice. For each
// slice, once the transcoding warps have freed its stage, the lane writes its
// row's width and base word and starts the row's 16*w exponent bytes (16-byte
// cp.async pieces); the stage's raw_full barrier then completes when all 128
// rows have done so and all their copies have landed. ESC: the lane also
// writes the block's exception-list length and address and copies the list's
// first kExcBytes bytes (the same for every slice of the block).
template <int MAXI, bool ESC>
__device__ void gemm_rows(const GemmParams<MAXI>& P, const GemmSmem& S, int pw, int lane) {
    GemmCtl& c = *S.ctl;
    const uint32_t R = P.ring;
    const uint32_t r = 32u * uint32_t(pw) + uint32_t(lane);
    const uint32_t raw_row = smem_addr(S.raw) + r * kExpPitch;
    UnitState U = {};
    RowState RS = {};
    UnitWalk wk;
    wk.start();
    uint32_t it = 0, sa = 0, slices = 0, row0 = 0;
    uint32_t rs = 0, round = 0;  // slice a: stage a % R, round a / R
    while (wk.u < P.total_units) {
        bool bad = false;
        if (sa == 0) {  // first slice of a unit: the row's first block, loaded here
            it = find_item(P, wk.u, it);
            U = unit_state(P, it);
            slices = U.cols / kSliceCols;
            row0 = uint32_t(wk.u - P.unit_begin[it]) * kTileRows;
            const uint64_t row = row0 + r;
            RS.valid = row < U.rows;
            set_width(RS, 0, 0);
            RS.left = 0;
            if (RS.valid) {
                const uint64_t el = row * U.cols;
                uint32_t h, off;
                uint64_t nx;
                load_block(U, el >> U.log2B, h, off, nx);
                bad |= !enter_block<ESC>(U, RS, row, el, h, off, nx);
            }
        } else if (RS.valid) {
            RS.left -= kSliceCols;
            RS.first = false;
            if (RS.left == 0)  // the slice starts the row's next block
                bad |= !enter_block<ESC>(U, RS, row0 + r, (RS.b + 1) << U.log2B, RS.nh, RS.noff,
                                         RS.nnx);
            else
                RS.src += 16u * RS.w;
        }
        if (bad) report(P.status, kStatusCorrupt);
        // the stage is free once the transcoding warps are done with slice a - R
        if (round > 0 && !gemm_wait_warp(&c.raw_empty[rs], (round - 1) & 1u, c, P.status)) break;
        const uint32_t w = RS.w;
        if (ESC) {
            const bool last = RS.valid && RS.left <= kSliceCols;
            S.meta[rs * kTileRows + r] =
                w | (RS.base << 8) | (RS.first ? kMetaFirst : 0u) | (last ? kMetaLast : 0u);
            const uint32_t xl = RS.valid ? RS.exc_len : 0u;
            const uint64_t xa = reinterpret_cast<uint64_t>(RS.exc);
            S.emeta[rs * kTileRows + r] = make_uint4(xl, uint32_t(xa), uint32_t(xa >> 32), 0u);
            const uint32_t xd = smem_addr(S.exc) + rs * kExcStage + r * kExcBytes;
#pragma unroll
            for (uint32_t j = 0; j < kExcBytes / 16; ++j)
                if (16u * (j + 1) <= xl) cp_async16(xd + 16u * j, RS.exc + 16u * j);
        } else {
            S.meta[rs * kTileRows + r] = w | (RS.base << 8);
        }
        const uint32_t d = raw_row + rs * kRawStage;
#pragma unroll
        for (uint32_t j = 0; j < 8; ++j)
            if (j < w) cp_async16(d + 16u * j, RS.src + 16u * j);
        cp_async_mbar_arrive(&c.raw_full[rs]);
        mbar_arrive(&c.raw_full[rs]);
        if (++sa == slices) {
            sa = 0;
            wk.next();
        }
        if (rs + 1 == R) rs = 0, ++round; else ++rs;
    }
    asm volatile("cp.async.wait_all;" ::: "memory");  // nothing lands after the block ends
}

// Slices the block works through (every role walks the same sequence).
template <int MAXI>
__device__ __forceinline__ uint32_t block_slices(const GemmParams<MAXI>& P) {
    uint32_t total = 0, it = 0;
    UnitWalk w;
    for (w.start(); w.u < P.total_units; w.next()) {
        it = find_item(P, w.u, it);
        total += P.item[it].cols / kSliceCols;
    }
    return total;
}

// Four values of w bits (a quad, bits [0, 4w) of q) -> four bytes base + v,
// for any w in 0..8: byte t takes bits [t*w, t*w + 8) of q, masked to w bits.
__device__ __forceinline__ uint32_t quad_bytes(uint32_t q, uint32_t w, uint32_t m1x4,
                                               uint32_t base4) {
    const uint32_t t1 = prmt(q, q >> w, 0x0040u);             // bytes 0, 1
    const uint32_t t2 = prmt(q >> (2u * w), q >> (3u * w), 0x4000u);  // bytes 2, 3
    return (prmt(t1, t2, 0x7610u) & m1x4) + base4;
}

// Octet of width W (compile time, at most 5) starting at byte q of a staged row:
// its eight values as bytes, value t in byte t % 4 of word t / 4. 8W <= 40
// bits starting at most 24 bits into a word lie in two words.
template <int W>
__device__ __forceinline__ void octet_bytes(const uint8_t* raw, uint32_t q, uint32_t& a,
                                            uint32_t& b) {
    const uint32_t* s32 = reinterpret_cast<const uint32_t*>(raw);
    const uint32_t i = q >> 2;
    const uint64_t v = ((uint64_t(s32[i + 1]) << 32) | s32[i]) >> ((q & 3u) * 8u);
    constexpr uint32_t kQuad = (1u << (4 * W)) - 1u;
    a = quad_to_bytes<W>(uint32_t(v) & kQuad);
    b = quad_to_bytes<W>(uint32_t(v >> (4 * W)) & kQuad);
}

// Transcoding warps: warp t owns rows 16t .. 16t+15 of every slice, eight
// lanes per row and four rows per step: step k takes rows 16t + k + 4*slot
// (slot = lane / 8), so the two rows of a half-warp are four apart and their
// loads and stores fall in complementary bank halves. Lane c = lane % 8 of a
// row takes octets o0 = 2c + (c / 4) and o1 = 2c + 1 - (c / 4) of its 16 --
// between them the two octets 2c and 2c + 1, so the lanes of a row hold its
// elements in lane order -- writing each octet's eight exponent bytes
// (base + code, no byte can carry: base + code <= 255 in a valid stream) with
// one 8-byte store.
// ESC: a code 2^w - 1 (1 <= w <= 7) is an escape, replaced by the next byte of
// the block's exception list: its index is the row's escapes in the block's
// earlier slices (kept per row in the lanes' registers), plus those of the
// row's lower lanes in this slice (a prefix sum over the row's eight lanes),
// plus those before it in the lane.
template <int MAXI, bool ESC>
__device__ void gemm_transcode(const GemmParams<MAXI>& P, const GemmSmem& S, int tw, int lane) {
    GemmCtl& c = *S.ctl;
    const uint32_t R = P.ring;
    // ESC: the lane's two octets in element order (8-byte loads, 16-byte stores:
    // 10 % faster there); plain: swapped in the upper half of the row's lanes so
    // that 4-byte accesses of two rows fall in complementary bank halves
    const uint32_t c8 = uint32_t(lane) & 7u, slot = uint32_t(lane) >> 3, pp = ESC ? 0u : c8 >> 2;
    const uint32_t o0 = 2u * c8 + pp, o1 = 2u * c8 + 1u - pp;
    const uint32_t row_base = 16u * uint32_t(tw) + 4u * slot;
    const uint32_t total = block_slices(P);
    uint32_t run[4] = {0u, 0u, 0u, 0u};  // ESC: the row's escapes in its block so far
    uint32_t rs = 0, round = 0;   // packed-exponent stage of slice g, and its round
    uint32_t es = 0, eround = 0;  // exponent-byte stage
    for (uint32_t g = 0; g < total; ++g) {
        if (!gemm_wait_warp(&c.raw_full[rs], round & 1u, c, P.status) ||
            (eround > 0 && !gemm_wait_warp(&c.e_empty[es], (eround - 1) & 1u, c, P.status)))
            break;
        const uint8_t* raw = S.raw + rs * kRawStage;
        const uint32_t* meta = S.meta + rs * kTileRows;
        const uint32_t e_stage = smem_addr(S.e + es * kEStage);
        // every load of the four steps first, the exponent words at their
        // width-4 places
        uint32_t mw[4], f[4][2];
#pragma unroll
        for (uint32_t k = 0; k < 4; ++k) {
            const uint32_t rr = row_base + k;
            mw[k] = meta[rr];
            const uint8_t* ep = raw + rr * kExpPitch;
            if (ESC) {
                const uint2 fw = *reinterpret_cast<const uint2*>(ep + 8u * c8);
                f[k][0] = fw.x;
                f[k][1] = fw.y;
            } else {
                f[k][0] = *reinterpret_cast<const uint32_t*>(ep + 4u * o0);
                f[k][1] = *reinterpret_cast<const uint32_t*>(ep + 4u * o1);
            }
        }
        bool bad = false;
        uint32_t fm[4] = {0u, 0u, 0u, 0u}, cnt4 = 0;  // ESC: escape flags and counts per step
        // One path per step of four rows, all four steps decided by one warp
        // reduction: bit k of all4 (all3) is set when every row of step k has
        // width 4 (3).
        uint32_t w4bits = 0, w3bits = 0;
#pragma unroll
        for (uint32_t k = 0; k < 4; ++k) {
            w4bits |= ((mw[k] & 0xFFu) == 4u ? 1u : 0u) << k;
            if (ESC) w3bits |= ((mw[k] & 0xFFu) == 3u ? 1u : 0u) << k;
        }
        const uint32_t all4 = __reduce_and_sync(0xFFFFFFFFu, w4bits);
        const uint32_t all3 = ESC ? __reduce_and_sync(0xFFFFFFFFu, w3bits) : 0u;
        if (!ESC && all4 == 0xFu) {
            // the common case: every row of the four steps at width 4, in
            // straight-line code (the four steps' work interleaves)
#pragma unroll
            for (uint32_t k = 0; k < 4; ++k) {
                const uint32_t rr = row_base + k;
                const uint32_t base4 = ((mw[k] >> 8) & 0xFFu) * 0x01010101u;
                uint32_t e[4];
#pragma unroll
                for (uint32_t h = 0; h < 2; ++h) {
                    const uint32_t ev = f[k][h] & 0x0F0F0F0Fu, od = (f[k][h] >> 4) & 0x0F0F0F0Fu;
                    e[2 * h] = prmt(ev, od, 0x5140u) + base4;
                    e[2 * h + 1] = prmt(ev, od, 0x7362u) + base4;
                }
                sts64(e_stage + rr * kExpPitch + 8u * o0, e[0], e[1]);
                sts64(e_stage + rr * kExpPitch + 8u * o1, e[2], e[3]);
            }
        } else {
#pragma unroll
        for (uint32_t k = 0; k < 4; ++k) {
            const uint32_t rr = row_base + k;
            const uint32_t w = mw[k] & 0xFFu, base = (mw[k] >> 8) & 0xFFu;
            const uint32_t base4 = ESC ? 0u : base * 0x01010101u;  // ESC: added after the escapes
            uint32_t e[4];
            if ((all4 >> k) & 1u) {
#pragma unroll
                for (uint32_t h = 0; h < 2; ++h) {
                    const uint32_t ev = f[k][h] & 0x0F0F0F0Fu, od = (f[k][h] >> 4) & 0x0F0F0F0Fu;
                    e[2 * h] = prmt(ev, od, 0x5140u) + base4;
                    e[2 * h + 1] = prmt(ev, od, 0x7362u) + base4;
                }
            } else if (ESC && ((all3 >> k) & 1u)) {  // escape-coded Gaussian blocks: width 3
                octet_bytes<3>(raw, rr * kExpPitch + 3u * o0, e[0], e[1]);
                octet_bytes<3>(raw, rr * kExpPitch + 3u * o1, e[2], e[3]);
            } else {
                const uint32_t* s32 = reinterpret_cast<const uint32_t*>(raw);
                const uint32_t m1x4 = ((1u << w) - 1u) * 0x01010101u;
                const uint32_t m4 = w == 8u ? 0xFFFFFFFFu : (1u << (4u * w)) - 1u;
#pragma unroll
                for (uint32_t h = 0; h < 2; ++h) {
                    uint32_t lo, hi;
                    fetch_octet(s32, rr * kExpPitch + (h ? o1 : o0) * w, lo, hi);
                    e[2 * h] = quad_bytes(lo & m4, w, m1x4, base4);
                    e[2 * h + 1] = quad_bytes(__funnelshift_rc(lo, hi, 4u * w) & m4, w, m1x4, base4);
                }
            }
            if (ESC) {
                // e holds codes: flag the escapes (counted below for all four
                // steps at once), add the base and store the bytes
                const uint32_t m = (1u << w) - 1u;
                // a code equals 2^w - 1 exactly when adding 0x80 - (2^w - 1) sets its
                // byte's top bit (codes are at most 2^w - 1: no carry leaves a byte)
                const bool windowed = w >= 1u && w <= 7u;
                const uint32_t esc_add = windowed ? (0x80u - m) * 0x01010101u : 0u;
                const uint32_t esc_det = windowed ? 0x80808080u : 0u;
                // bit 4j + t of fm[k]: byte t of e[j] is an escape, so the lane's 16
                // elements are in bit order. A word's four flags (bits 7, 15, 23,
                // 31) gather into bits 24..27 of (flags >> 7) * 0x01020408: every
                // partial product lands on a bit of its own, so nothing carries.
                uint32_t f16 = 0;
#pragma unroll
                for (uint32_t j = 0; j < 4; ++j) {
                    const uint32_t fl = (e[j] + esc_add) & esc_det;
                    f16 |= (((fl >> 7) * 0x01020408u) >> 24) << (4u * j);
                }
                fm[k] = f16;
                cnt4 |= uint32_t(__popc(f16)) << (8u * k);
                const uint32_t b4 = base * 0x01010101u;  // base + code <= 255: no carries
#pragma unroll
                for (uint32_t j = 0; j < 4; ++j) e[j] += b4;
                // escapes still as base + 2^w - 1: the patch below overwrites them
                sts128(e_stage + rr * kExpPitch + 16u * c8, e[0], e[1], e[2], e[3]);
            } else {
                sts64(e_stage + rr * kExpPitch + 8u * o0, e[0], e[1]);
                sts64(e_stage + rr * kExpPitch + 8u * o1, e[2], e[3]);
            }
        }
        }
        if (ESC) {
            // The four steps' escape counts, one byte per step, scanned over the
            // row's eight lanes at once (a row has at most 128 escapes in a
            // slice: no byte carries into the next).
            uint32_t incl4 = cnt4;
#pragma unroll
            for (uint32_t d = 1; d < 8; d <<= 1) {
                const uint32_t y = __shfl_up_sync(0xFFFFFFFFu, incl4, d, 8);
                if (c8 >= d) incl4 += y;
            }
            const uint32_t tot4 = __shfl_sync(0xFFFFFFFFu, incl4, 7, 8);
#pragma unroll
            for (uint32_t k = 0; k < 4; ++k) {
                const uint32_t rr = row_base + k;
                const uint32_t w = mw[k] & 0xFFu, base = (mw[k] >> 8) & 0xFFu;
                const uint32_t m = (1u << w) - 1u;
                const uint32_t cnt = (cnt4 >> (8u * k)) & 0xFFu;
                const uint32_t incl = (incl4 >> (8u * k)) & 0xFFu;
                const uint32_t row_total = (tot4 >> (8u * k)) & 0xFFu;
                if (mw[k] & kMetaFirst) run[k] = 0;
                const bool last = (mw[k] & kMetaLast) != 0u;
                uint32_t f16 = fm[k];
                if (__any_sync(0xFFFFFFFFu, f16 != 0u || last)) {
                    const uint4 em = S.emeta[rs * kTileRows + rr];
                    const uint8_t* xg = reinterpret_cast<const uint8_t*>(
                        (uint64_t(em.z) << 32) | uint64_t(em.y));
                    const uint8_t* xs = S.exc + rs * kExcStage + rr * kExcBytes;
                    const uint32_t row_at = e_stage + rr * kExpPitch + 16u * c8;
                    uint32_t idx = run[k] + incl - cnt;  // the lane's first exception
                    // one pass over the lane's escapes in element order (one loop
                    // for all sixteen elements: a warp runs as many rounds as its
                    // lane with the most escapes has)
                    while (f16) {
                        const uint32_t t = __ffs(int(f16)) - 1u;
                        uint32_t x = 0;
                        if (idx < em.x) x = idx < kExcBytes ? xs[idx] : xg[idx];
                        else bad = true;
                        bad |= ((x - base) & 0xFFu) < m;  // an exception inside the window
                        sts8(row_at + t, x);
                        ++idx;
                        f16 &= f16 - 1u;
                    }
                    // the block's last slice: the list holds exactly its escapes
                    // (up to the payload's 15 bytes of padding)
                    if (last && c8 == 7u)
                        bad |= run[k] + row_total > em.x || em.x - (run[k] + row_total) > 15u;
                }
                run[k] += row_total;
            }
        }
        if (ESC && bad) report(P.status, kStatusCorrupt);
        __syncwarp();
        if (lane == 0) {
            mbar_arrive(&c.raw_empty[rs]);
            mbar_arrive(&c.e_full[es]);
        }
        if (++rs == R) rs = 0, ++round;
        if (++es == kERing) es = 0, ++eround;
    }
}

// Four sign+mantissa bytes s and four exponent bytes e -> four BF16 words in
// two 32-bit words (element 0 in the low half of o0):
//   BF16 = (s & 0x80) << 8 | e << 7 | (s & 0x7F)
// the exponent bytes spread into the two 16-bit halves by a byte permute and
// shifted by a multiply-add that also adds the masked sign+mantissa bits (no
// carries: the fields are disjoint). The multiply-add runs on the FMA pipe,
// which the writing warps otherwise leave idle while their ALU pipe is the
// busy one; the all-ALU form (two bit-selects and two permutes) was 7 % slower.
__device__ __forceinline__ void merge4(uint32_t s, uint32_t e, uint32_t& o0, uint32_t& o1) {
    o0 = prmt(e, 0u, 0x4140u) * 128u + (prmt(s, 0u, 0x1100u) & 0x807F807Fu);
    o1 = prmt(e, 0u, 0x4342u) * 128u + (prmt(s, 0u, 0x3322u) & 0x807F807Fu);
}

// Writing warps: lane l of writing warp i owns row 32q + l (q = i % 4, the
// tensor memory lanes its warp rank may access) and columns 64h .. 64h+63 of
// every slice (h = i / 4). It loads the row's 64 sign+mantissa bytes from the
// swizzled mantissa stage and its 64 exponent bytes, merges them into BF16
// and stores them into the slice's A stage in tensor memory: lane = row,
// column k = weights 2k and 2k+1 of the row, the layout tcgen05.mma reads A in.
template <int MAXI>
__device__ void gemm_write(const GemmParams<MAXI>& P, const GemmSmem& S, int wi, int lane) {
    GemmCtl& c = *S.ctl;
    const uint32_t R = P.ring;
    const uint32_t q = uint32_t(wi) & 3u, kh = uint32_t(wi) >> 2;
    const uint32_t r = 32u * q + uint32_t(lane);
    const uint32_t sw = r & 7u;
    const uint32_t man_row = smem_addr(S.man) + r * 128u;
    const uint32_t e_row = smem_addr(S.e) + r * kExpPitch + 64u * kh;
    const uint32_t t_lane = c.tmem_base + ((32u * q) << 16) + kACol0 + 32u * kh;
    const uint32_t total = block_slices(P);
    uint32_t rs = 0, round = 0, es = 0, eround = 0, as = 0, around = 0;
    for (uint32_t g = 0; g < total; ++g) {
        if (!gemm_wait_warp(&c.man_full[rs], round & 1u, c, P.status) ||
            !gemm_wait_warp(&c.e_full[es], eround & 1u, c, P.status))
            break;
        const uint32_t man = man_row + rs * kManStage, ex = e_row + es * kEStage;
        uint4 sm[4], ev[4];
#pragma unroll
        for (uint32_t i = 0; i < 4; ++i) {
            sm[i] = lds128(man + (((4u * kh + i) ^ sw) << 4));
            ev[i] = lds128(ex + 16u * i);
        }
        if (around > 0 && !gemm_wait_warp(&c.a_empty[as], (around - 1) & 1u, c, P.status)) break;
        tc_fence_after();
#pragma unroll
        for (uint32_t h = 0; h < 2; ++h) {
            uint32_t v[16];
#pragma unroll
            for (uint32_t i = 0; i < 2; ++i) {
                const uint4 s4 = sm[2 * h + i], e4 = ev[2 * h + i];
                merge4(s4.x, e4.x, v[8 * i + 0], v[8 * i + 1]);
                merge4(s4.y, e4.y, v[8 * i + 2], v[8 * i + 3]);
                merge4(s4.z, e4.z, v[8 * i + 4], v[8 * i + 5]);
                merge4(s4.w, e4.w, v[8 * i + 6], v[8 * i + 7]);
            }
            tmem_st16(t_lane + as * kACols + 16u * h, v);
        }
        tmem_wait_st();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) {
            mbar_arrive(&c.man_empty[rs]);
            mbar_arrive(&c.e_empty[es]);
            mbar_arrive(&c.a_full[as]);
        }
        if (++rs == R) rs = 0, ++round;
        if (++es == kERing) es = 0, ++eround;
        if (++as == kARing) as = 0, ++around;
    }
}

// ---------------------------------------------------------------------------
// MMA issue (one thread)
// ---------------------------------------------------------------------------
template <int MAXI>
__device__ void gemm_mma(const GemmParams<MAXI>& P, const GemmSmem& S) {
    GemmCtl& c = *S.ctl;
    // The single issuing thread is the pace-setter: an MMA of M = 128, K = 16
    // takes the tensor pipe some 50 cycles for N <= 64, and every instruction
    // the thread spends between two MMAs delays the next one. So everything
    // but a few adds is computed before the slice's eight MMAs: the two
    // activation panels' descriptors (per slice), the accumulator column of
    // each MMA (per unit) and the accumulate flags (per slice).
    const uint32_t idesc = bf16_idesc(kTileRows, P.nt);
    const uint32_t x0 = smem_addr(S.x);
    const uint32_t xstage = P.nt * 256, xpanel16 = P.nt * 8;  // a panel in 16-byte units
    const uint32_t amask = P.nacc - 1u;
    uint32_t j = 0, it = 0, as = 0, around = 0, xs = 0, xround = 0;
    bool issued = false;
    UnitWalk w;
    for (w.start(); w.u < P.total_units; w.next(), ++j) {
        it = find_item(P, w.u, it);
        const uint32_t slices = P.item[it].cols / kSliceCols;
        const uint32_t buf = P.nbuf == 2 ? (j & 1u) : 0u, use = P.nbuf == 2 ? (j >> 1) : j;
        if (use >= 1 && !gemm_wait(&c.acc_empty[buf], (use - 1) & 1u, c, P.status)) break;
        tc_fence_after();
        // consecutive MMAs go to different accumulators, so that they do not
        // wait for one another's results
        uint32_t d[8];
        const uint32_t d0 = c.tmem_base + buf * P.nacc * P.nt;
#pragma unroll
        for (uint32_t kk = 0; kk < 8; ++kk) d[kk] = d0 + (kk & amask) * P.nt;
        // accumulate flags of the unit's first slice: the first MMA into each
        // accumulator overwrites it
        const uint32_t first_mask = 0xFFu & ~((2u << amask) - 1u);
        bool ok = true;
        for (uint32_t s = 0; s < slices; ++s) {
            if (!gemm_wait(&c.a_full[as], around & 1u, c, P.status) ||
                !gemm_wait(&c.x_full[xs], xround & 1u, c, P.status)) {
                ok = false;
                break;
            }
            tc_fence_after();
            const uint32_t a = c.tmem_base + kACol0 + as * kACols;
            const uint64_t xd0 = sw128_desc(x0 + xs * xstage);
            const uint64_t xd1 = xd0 + xpanel16;
            const uint32_t en = s == 0 ? first_mask : 0xFFu;
#pragma unroll
            for (uint32_t kk = 0; kk < kSliceCols / 16; ++kk)  // 16 BF16 = 32 bytes = 2 units along K
                umma_bf16_ts(d[kk], a + 8u * kk, (kk < 4 ? xd0 : xd1) + 2u * (kk & 3u), idesc,
                             en & (1u << kk));
            issued = true;
            umma_commit(&c.a_empty[as]);
            umma_commit(&c.x_empty[xs]);
            if (++as == kARing) as = 0, ++around;
            if (++xs == P.xring) xs = 0, ++xround;
        }
        if (!ok) break;
        umma_commit(&c.acc_full[buf]);
    }
    // Every MMA has finished reading its operands and writing TMEM before the block ends.
    if (issued) {
        umma_commit(&c.drain);
        mbar_wait(&c.drain, 0, nullptr);
    }
}

// ---------------------------------------------------------------------------
// epilogue warps: TMEM lane quarter q = warp % 4 holds rows 32q .. 32q+31 of the
// unit; lane l reads its row's nt FP32 columns 16 at a time and writes
// Y[t][row0 + 32q + l] (32 consecutive floats per warp and token).
// ---------------------------------------------------------------------------
template <int MAXI>
__device__ void gemm_epilogue(const GemmParams<MAXI>& P, const GemmSmem& S, int warp, int lane) {
    GemmCtl& c = *S.ctl;
    const uint32_t q = uint32_t(warp) & 3u;
    uint32_t j = 0, it = 0;
    UnitWalk w;
    for (w.start(); w.u < P.total_units; w.next(), ++j) {
        it = find_item(P, w.u, it);
        const GemvItem& I = P.item[it];
        const uint32_t row = uint32_t(w.u - P.unit_begin[it]) * kTileRows + 32u * q + uint32_t(lane);
        const uint32_t buf = P.nbuf == 2 ? (j & 1u) : 0u, use = P.nbuf == 2 ? (j >> 1) : j;
        if (!gemm_wait_warp(&c.acc_full[buf], use & 1u, c, P.status, 512)) return;
        tc_fence_after();
        const uint32_t taddr = c.tmem_base + ((32u * q) << 16) + buf * P.nacc * P.nt;
        for (uint32_t cg = 0; cg < P.nt; cg += 16) {
            // the unit's accumulators summed in a fixed order: the same bits every run
            uint32_t v[16];
            tmem_ld16(taddr + cg, v);
            float y[16];
#pragma unroll
            for (uint32_t i = 0; i < 16; ++i) y[i] = __uint_as_float(v[i]);
            for (uint32_t a = 1; a < P.nacc; ++a) {
                tmem_ld16(taddr + a * P.nt + cg, v);
#pragma unroll
                for (uint32_t i = 0; i < 16; ++i) y[i] += __uint_as_float(v[i]);
            }
            if (row < I.rows) {
#pragma unroll
                for (uint32_t i = 0; i < 16; ++i)
                    if (cg + i < P.tokens) I.y[uint64_t(cg + i) * I.rows + row] = y[i];
            }
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&c.acc_empty[buf]);
    }
}

// ESC: escape-coded streams. The two stream kinds are separate kernels, so
// that each gets its own register allocation and code layout (the escape
// handling would otherwise shape the plain kernel's).
template <int MAXI, bool ESC>
__global__ void __launch_bounds__(kGemmThreads, 1)
    gemm_kernel(const __grid_constant__ GemmParams<MAXI> P) {
    extern __shared__ __align__(1024) unsigned char smem_raw[];
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    // carve shared memory (1024-aligned regions)
    const uint32_t base = smem_addr(smem_raw);
    uint8_t* p = smem_raw + ((1024u - (base & 1023u)) & 1023u);
    GemmSmem S;
    S.ctl = reinterpret_cast<GemmCtl*>(p);
    p += 1024;
    S.x = p;
    p += P.xring * P.nt * 256;
    S.man = p;
    p += P.ring * kManStage;
    S.raw = p;
    p += P.ring * kRawStage;
    S.e = p;
    p += kERing * kEStage;
    S.meta = reinterpret_cast<uint32_t*>(p);
    p += P.ring * kMetaStage;
    S.exc = p;  // escape-coded streams only (the layout's size counts them then)
    p += P.escape ? P.ring * kExcStage : 0u;
    S.emeta = reinterpret_cast<uint4*>(p);
    GemmCtl& c = *S.ctl;
    if (tid == 0) {
        for (uint32_t s = 0; s < kMaxRing; ++s) {
            mbar_init(&c.man_full[s], 1);
            mbar_init(&c.man_empty[s], kWrtWarps);
            mbar_init(&c.raw_full[s], 32 * kRowWarps);
            mbar_init(&c.raw_empty[s], kTrWarps);
        }
        for (uint32_t s = 0; s < kERing; ++s) {
            mbar_init(&c.e_full[s], kTrWarps);
            mbar_init(&c.e_empty[s], kWrtWarps);
        }
        for (uint32_t s = 0; s < kARing; ++s) {
            mbar_init(&c.a_full[s], kWrtWarps);
            mbar_init(&c.a_empty[s], 1);
        }
        for (uint32_t s = 0; s < kMaxXRing; ++s) {
            mbar_init(&c.x_full[s], 1);
            mbar_init(&c.x_empty[s], 1);
        }
        for (int s = 0; s < 2; ++s) {
            mbar_init(&c.acc_full[s], 1);
            mbar_init(&c.acc_empty[s], kEpiWarps);
        }
        mbar_init(&c.drain, 1);
        c.abort = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    if (warp == kMmaWarp) {  // all of tensor memory: two accumulators and the A stages
        asm volatile(
            "tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                smem_addr(&c.tmem_base)),
            "r"(512)
            : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();

    if (warp == kProducerWarp) {
        if (lane == 0) gemm_produce<MAXI>(P, S);
    } else if (warp == kMmaWarp) {
        if (lane == 0) gemm_mma<MAXI>(P, S);
    } else if (warp == kXWarp) {
        if (lane == 0) gemm_load_x<MAXI>(P, S);
    } else if (warp >= kEpiWarp0 && warp < kEpiWarp0 + kEpiWarps) {
        gemm_epilogue<MAXI>(P, S, warp, lane);
    } else if (warp >= kWrtWarp0 && warp < kWrtWarp0 + kWrtWarps) {
        gemm_write<MAXI>(P, S, warp - kWrtWarp0, lane);
    } else if (warp >= kTrWarp0 && warp < kTrWarp0 + kTrWarps) {
        gemm_transcode<MAXI, ESC>(P, S, warp - kTrWarp0, lane);
    } else if (warp >= kRowWarp0) {
        gemm_rows<MAXI, ESC>(P, S, warp - kRowWarp0, lane);
    }

    tc_fence_before();
    __syncthreads();
    if (warp == kMmaWarp) {
        tc_fence_after();
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(c.tmem_base),
                     "r"(512)
                     : "memory");
    }
}

// ---------------------------------------------------------------------------
// host side
// ---------------------------------------------------------------------------
PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
    static std::once_flag once;
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    std::call_once(once, [] {
        void* f = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &f, 12000, cudaEnableDefault,
                                             &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(f);
    });
    return fn;
}

template <int MAXI>
cudaError_t gemm_launch(const GemvItem* items, uint32_t count, uint32_t tokens, bool escape,
                        int32_t* status, cudaStream_t stream) {
    static_assert(sizeof(GemmParams<MAXI>) <= 32000, "launch parameters exceed the limit");
    PFN_cuTensorMapEncodeTiled_v12000 enc = encode_fn();
    if (enc == nullptr) return cudaErrorNotSupported;
    GemmParams<MAXI> p;
    memset(&p, 0, sizeof(p));
    p.status = status;
    p.count = count;
    p.tokens = tokens;
    p.nt = (tokens + 15u) & ~15u;
    p.escape = escape ? 1u : 0u;
    gemm_rings(p.nt, escape, &p.ring, &p.xring);
    // accumulators below column kACol0: two units in flight when they fit with
    // at least two accumulators each, else one unit with two
    p.nbuf = 4u * p.nt <= kACol0 ? 2u : 1u;
    p.nacc = 1u;
    while (p.nacc < 4u && p.nbuf * 2u * p.nacc * p.nt <= kACol0) p.nacc *= 2u;
    if (gemm_smem_bytes(p.nt, p.ring, p.xring, escape) > kSmemLimit) return cudaErrorInvalidValue;
    // Units are numbered longest first (matrices by decreasing column count,
    // ties in the caller's order) for the blocks' snake walk.
    uint32_t order[MAXI];
    for (uint32_t i = 0; i < count; ++i) order[i] = i;
    std::stable_sort(order, order + count,
                     [&](uint32_t a, uint32_t b) { return items[a].cols > items[b].cols; });
    uint64_t units = 0;
    for (uint32_t i = 0; i < count; ++i) {
        const GemvItem& I = items[order[i]];
        p.item[i] = I;
        p.unit_begin[i] = units;
        units += (uint64_t(I.rows) + kTileRows - 1) / kTileRows;
        if (I.rows == 0) continue;
        const Layout L = make_layout(uint64_t(I.rows) * I.cols, I.block);
        {
            const cuuint64_t dims[2] = {I.cols, I.rows};
            const cuuint64_t strides[1] = {I.cols};
            const cuuint32_t box[2] = {kSliceCols, kTileRows};
            const cuuint32_t estr[2] = {1, 1};
            if (enc(&p.man_map[i], CU_TENSOR_MAP_DATA_TYPE_UINT8, 2,
                    const_cast<uint8_t*>(I.stream + L.off_man), dims, strides, box, estr,
                    CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                    CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                    CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
                return cudaErrorInvalidValue;
        }
        {
            const cuuint64_t dims[2] = {I.cols, tokens};
            const cuuint64_t strides[1] = {uint64_t(I.cols) * 2};
            const cuuint32_t box[2] = {64, p.nt};
            const cuuint32_t estr[2] = {1, 1};
            if (enc(&p.x_map[i], CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<uint16_t*>(I.x),
                    dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                    CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                    CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
                return cudaErrorInvalidValue;
        }
    }
    p.unit_begin[count] = units;
    p.total_units = units;
    if (units == 0) return cudaSuccess;

    static std::mutex mu;
    static int sms_of[64];
    static uint32_t smem_set[2][64];  // per stream kind
    int dev = 0;
    cudaError_t err = cudaGetDevice(&dev);
    if (err != cudaSuccess) return err;
    if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
    const uint32_t smem = gemm_smem_bytes(p.nt, p.ring, p.xring, escape);
    const auto kernel = escape ? gemm_kernel<MAXI, true> : gemm_kernel<MAXI, false>;
    {
        std::lock_guard<std::mutex> lock(mu);
        if (sms_of[dev] == 0) {
            err = cudaDeviceGetAttribute(&sms_of[dev], cudaDevAttrMultiProcessorCount, dev);
            if (err != cudaSuccess) return err;
        }
        if (smem_set[escape ? 1 : 0][dev] < smem) {
            err = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       int(kSmemLimit));
            if (err != cudaSuccess) return err;
            smem_set[escape ? 1 : 0][dev] = kSmemLimit;
        }
    }
    const uint64_t cap = uint64_t(sms_of[dev]);
    const unsigned grid = unsigned(units < cap ? units : cap);
    kernel<<<grid, kGemmThreads, smem, stream>>>(p);
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_gemm(const GemvItem* items, uint32_t count, uint32_t tokens, bool escape,
                        int32_t* status, cudaStream_t stream) {
    if (tokens < 1 || tokens > kMaxGemmTokens) return cudaErrorInvalidValue;
    constexpr uint32_t kBatch = kGemmBatchMax;
    if (count == 1) return gemm_launch<1>(items, 1, tokens, escape, status, stream);
    for (uint32_t i = 0; i < count; i += kBatch) {
        const uint32_t c = min(kBatch, count - i);
        const cudaError_t err = gemm_launch<kBatch>(items + i, c, tokens, escape, status, stream);
        if (err != cudaSuccess) return err;
    }
    return cudaSuccess;
}

}  // namespace wc
