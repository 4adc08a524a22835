// wc_gemm.cu -- fused decompression and matrix products on the sm_100a tensor cores.
//
// Y[t][r] = sum_c W[r][c] * X[t][c] for t < tokens (1..128), where the BF16
// weight matrix W (rows x cols, row-major) is held only as a WCB1 stream: each
// 128 x 128 slice of W is decoded into shared memory and fed to the tensor
// cores from there, so decoded weights never touch HBM ("ZipServ: Fast and
// Memory-Efficient LLM Inference with Hardware-Aware Lossless Compression",
// Abstract: decompression fused into the matrix product, load compressed and
// compute decompressed).
//
// One thread block per SM, persistent. A unit is 128 consecutive rows of one
// matrix (the MMA's M) times all tokens (its N, padded to a multiple of 16),
// swept over cols in slices of 128:
//   - one thread starts each slice's mantissa bytes (one 2-D TMA load,
//     128-byte swizzled) and another its activations (two 2-D TMA loads);
//   - four preparing warps, a few slices ahead, check each row's block
//     header and offset and fetch the row's exponent bytes (a 128-column slice
//     of a row is 16 whole octets of one block, 16*w contiguous bytes; 16-byte
//     cp.async pieces);
//   - sixteen decoding warps own 8 rows each and turn the staged bytes into
//     BF16 weights in the K-major 128-byte-swizzled layout the MMA reads;
//   - one thread issues tcgen05.mma (BF16 x BF16 -> FP32, M = 128, K = 16) into
//     one of two accumulators in tensor memory;
//   - four epilogue warps move a finished accumulator out with tcgen05.ld and
//     write Y while the next unit accumulates in the other one.
// Hand-offs use mbarriers; every wait is bounded by the device timer, after
// which the block stops and reports WC_ERR_TIMEOUT. Each unit sums its row in
// the same order on every run, so Y is reproducible bit for bit.
#include <cuda.h>
#include <cudaTypedefs.h>

#include <string.h>

#include <algorithm>
#include <mutex>

#include "wc_decode_core.cuh"

namespace wc {
namespace {

constexpr uint32_t kTileRows = 128;    // MMA M
constexpr uint32_t kSliceCols = 128;   // columns per pipeline slice (8 MMAs of K = 16)
constexpr uint32_t kExpPitch = 144;    // staged exponent bytes per row (16*w <= 128, +16 spreads banks)
constexpr uint32_t kManStage = kTileRows * kSliceCols;      // 16 KB
constexpr uint32_t kExpStage = kTileRows * kExpPitch;       // 18 KB
constexpr uint32_t kMetaStage = kTileRows * 4;              // w | base << 8 per row
constexpr uint32_t kAStage = kTileRows * kSliceCols * 2;    // 32 KB: two 64-column panels
constexpr uint32_t kAPanel = kTileRows * 128;               // 128 rows x 128 bytes
constexpr uint32_t kMaxRawStages = 3;
constexpr uint32_t kSmemLimit = 232448;                     // 227 KB per block

constexpr int kProducerWarp = 0;
constexpr int kMmaWarp = 1;
constexpr int kEpiWarp0 = 2;   // warps 2..5: warp % 4 covers the four TMEM lane quarters
constexpr int kEpiWarps = 4;
constexpr int kDecWarp0 = 6;
constexpr int kDecWarps = 16;
constexpr int kXWarp = kDecWarp0 + kDecWarps;    // 22: activation loader
constexpr int kPrepWarp0 = kXWarp + 1;           // 23..26: one lane per row of the tile
constexpr int kPrepWarps = 4;
constexpr int kGemmThreads = 32 * (kPrepWarp0 + kPrepWarps);  // 864

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
    uint32_t raw_stages;  // 2 or 3, whatever fits in shared memory
    uint32_t tmem_cols;   // power of two >= 2 * nt
    uint32_t pad;
};

// Shared memory, carved at run time (sizes depend on nt and raw_stages). The
// big regions start 1024-byte aligned, as the 128-byte swizzle pattern repeats
// every 8 rows of 128 bytes and is a function of the address.
struct GemmCtl {
    unsigned long long raw_full[kMaxRawStages], raw_empty[kMaxRawStages];
    unsigned long long exp_full[kMaxRawStages];  // a stage's exponent bytes and row words are in
    unsigned long long a_full[2], x_full[2], ax_empty[2];
    unsigned long long acc_full[2], acc_empty[2];
    unsigned long long drain;
    uint32_t tmem_base;
    int abort;
};

struct GemmSmem {
    GemmCtl* ctl;
    uint8_t* a;     // 2 stages
    uint8_t* x;     // 2 stages of nt * 256 bytes
    uint8_t* man;   // raw_stages stages
    uint8_t* exp;
    uint32_t* meta;  // per stage: w | base << 8 of each row
};

__host__ __device__ inline uint32_t gemm_smem_bytes(uint32_t nt, uint32_t raw_stages) {
    return 1024 + 1024 /* control */ + 2 * kAStage + 2 * nt * 256 +
           raw_stages * (kManStage + kExpStage + kMetaStage);
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

__device__ __forceinline__ void umma_bf16(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc,
                                          uint32_t idesc, uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
        "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
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

// 2-D tiled TMA load (no multicast) of the box at (c0, c1), completing on `bar`.
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

__device__ __forceinline__ void sts128(uint32_t saddr, uint4 v) {
    asm volatile("st.shared.v4.u32 [%0], {%1,%2,%3,%4};" ::"r"(saddr), "r"(v.x), "r"(v.y),
                 "r"(v.z), "r"(v.w)
                 : "memory");
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
// into a free raw stage; and the container header of each matrix, once.
// ---------------------------------------------------------------------------
template <int MAXI>
__device__ void gemm_produce(const GemmParams<MAXI>& P, const GemmSmem& S) {
    GemmCtl& c = *S.ctl;
    const uint32_t R = P.raw_stages;
    int raw_issued[kMaxRawStages] = {-1, -1, -1};  // to drain if the block stops early
    bool ok = true;
    uint32_t g = 0, rs = 0, round = 0;  // slice g goes to raw stage rs = g % R in round g / R
    for (Cursor cur = cursor_first(P); cur.valid;
         cur = cursor_next(P, cur), ++g, rs = rs + 1 == R ? (++round, 0u) : rs + 1) {
        const GemvItem& I = P.item[cur.it];
        if (cur.row0 == 0 && cur.s == 0) {
            DecodeItem d;
            d.stream = I.stream;
            d.stream_bytes = I.stream_bytes;
            check_container(d, make_layout(uint64_t(I.rows) * I.cols, I.block), P.status);
        }
        if (round > 0 && !gemm_wait(&c.raw_empty[rs], (round - 1) & 1u, c, P.status, 256)) {
            ok = false;
            break;
        }
        mbar_arrive_expect_tx(&c.raw_full[rs], kManStage);
        tma_load_2d(S.man + rs * kManStage, &P.man_map[cur.it], int32_t(cur.s * kSliceCols),
                    int32_t(cur.row0), &c.raw_full[rs]);
        raw_issued[rs] = int(round);
    }
    // Stopped early: let the copies already started land before the block exits.
    if (!ok)
        for (uint32_t k = 0; k < R; ++k)
            if (raw_issued[k] >= 0) mbar_wait(&c.raw_full[k], uint32_t(raw_issued[k]) & 1u, nullptr);
}

// ---------------------------------------------------------------------------
// activation loader (one thread): X for slice g goes into stage g % 2 once the
// MMAs of slice g - 2 have finished reading it
// ---------------------------------------------------------------------------
template <int MAXI>
__device__ void gemm_load_x(const GemmParams<MAXI>& P, const GemmSmem& S) {
    GemmCtl& c = *S.ctl;
    int x_issued[2] = {-1, -1};
    bool ok = true;
    uint32_t g = 0;
    for (Cursor cur = cursor_first(P); cur.valid; cur = cursor_next(P, cur), ++g) {
        const uint32_t xs = g & 1u;
        if (g >= 2 && !gemm_wait(&c.ax_empty[xs], ((g >> 1) - 1) & 1u, c, P.status, 256)) {
            ok = false;
            break;
        }
        const int32_t k0 = int32_t(cur.s * kSliceCols);
        uint8_t* xd = S.x + xs * P.nt * 256;
        mbar_arrive_expect_tx(&c.x_full[xs], P.nt * 256);
        tma_load_2d(xd, &P.x_map[cur.it], k0, 0, &c.x_full[xs]);
        tma_load_2d(xd + P.nt * 128, &P.x_map[cur.it], k0 + 64, 0, &c.x_full[xs]);
        x_issued[xs] = int(g >> 1);
    }
    if (!ok)
        for (int k = 0; k < 2; ++k)
            if (x_issued[k] >= 0) mbar_wait(&c.x_full[k], uint32_t(x_issued[k]) & 1u, nullptr);
}

// ---------------------------------------------------------------------------
// preparing and decoding warps. A slice is 128 rows x 128 columns.
//
// Four preparing warps run a few slices ahead, one lane per row: a lane checks
// its row's block header and offset when the row enters a block (the header
// was loaded when the row entered the previous block), writes the row's width
// and base to the slice's stage, and fetches the row's 16*w exponent bytes
// (16-byte cp.async pieces). An mbarrier per stage hands the staged bytes
// over; it completes once every row's lane has arrived and all their copies
// have landed.
//
// Sixteen decoding warps own 8 rows each and turn the staged bytes into BF16
// weights in the K-major 128-byte-swizzled layout the MMA reads.
// ---------------------------------------------------------------------------
static_assert(kDecWarps * 8 == int(kTileRows), "each decoding warp owns 8 rows");

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
    bool valid;
};

__device__ __forceinline__ void set_width(RowState& R, uint32_t w, uint32_t base) {
    R.w = w;
    R.base = base;
}

// Decode constants of a row from its width and base, in the form decode_octet
// takes: t0 = {row offset, w, 2w, 4w}, t1 = {pair masks, 2w-bit mask, 4w-bit
// mask, base << 7 in both 16-bit lanes}.
__device__ __forceinline__ void row_constants(uint32_t row_off, uint32_t w, uint32_t base,
                                              uint4& t0, uint4& t1) {
    const uint32_t m1 = (1u << w) - 1u;
    t0 = make_uint4(row_off, w, 2 * w, 4 * w);
    t1 = make_uint4(m1 | (m1 << 16), (1u << (2 * w)) - 1u,
                    w == 8u ? 0xFFFFFFFFu : (1u << (4 * w)) - 1u, base * 0x00800080u);
}

// Unit-level constants of the slice being prepared.
struct UnitState {
    const uint8_t* stream;
    uint64_t stream_bytes, n, nb, off_exp;
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
__device__ __forceinline__ bool enter_block(const UnitState& U, RowState& R, uint64_t row,
                                            uint64_t el, uint32_t h, uint32_t off, uint64_t nx) {
    const uint64_t b = el >> U.log2B;
    const uint32_t ob = uint32_t(el) & (U.block - 1u);  // the slice's offset in the block
    const uint64_t len = min(uint64_t(U.block), U.n - (b << U.log2B));
    uint32_t w = h >> 8, base = h & 0xFFu;
    bool bad = w > 8u || (w == 8u && base != 0u);
    const uint64_t sb = 16ull * off, end = sb + ((len + 7) >> 3) * min(w, 8u);
    if (ob == 0) bad |= end != nx;
    bad |= U.off_exp + end > U.stream_bytes;
    if (bad) w = base = 0;
    R.b = b;
    R.left = uint32_t(len) - ob;
    R.src = U.stream + U.off_exp + sb + (ob >> 3) * w;
    set_width(R, w, base);
    // the row continues into block b + 1 inside this unit's columns?
    if (((b + 1) << U.log2B) < (row + 1) * uint64_t(U.cols)) load_block(U, b + 1, R.nh, R.noff, R.nnx);
    return !bad;
}

// Preparing warps: lane l of preparing warp p owns row 32p + l of every slice.
// For each slice, once the decoding warps have freed its stage, the lane writes
// its row's width and base word and starts the row's 16*w exponent bytes
// (16-byte cp.async pieces); the stage's exp_full barrier then completes when
// all 128 rows have done so and all their copies have landed.
template <int MAXI>
__device__ void gemm_prepare(const GemmParams<MAXI>& P, const GemmSmem& S, int pw, int lane) {
    GemmCtl& c = *S.ctl;
    const uint32_t R = P.raw_stages;
    const uint32_t r = 32u * uint32_t(pw) + uint32_t(lane);
    const uint32_t exp_row = smem_addr(S.exp) + r * kExpPitch;
    UnitState U = {};
    RowState RS = {};
    UnitWalk wk;
    wk.start();
    uint32_t it = 0, sa = 0, slices = 0, row0 = 0;
    uint32_t rs = 0, round = 0;  // slice a: raw stage a % R, round a / R
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
                bad |= !enter_block(U, RS, row, el, h, off, nx);
            }
        } else if (RS.valid) {
            RS.left -= kSliceCols;
            if (RS.left == 0)  // the slice starts the row's next block
                bad |= !enter_block(U, RS, row0 + r, (RS.b + 1) << U.log2B, RS.nh, RS.noff, RS.nnx);
            else
                RS.src += 16u * RS.w;
        }
        if (bad) report(P.status, kStatusCorrupt);
        // the stage is free once the decoding warps are done with slice a - R
        if (round > 0 && !gemm_wait_warp(&c.raw_empty[rs], (round - 1) & 1u, c, P.status)) break;
        const uint32_t w = RS.w;
        S.meta[rs * kTileRows + r] = w | (RS.base << 8);
        const uint32_t d = exp_row + rs * kExpStage;
#pragma unroll
        for (uint32_t j = 0; j < 8; ++j)
            if (j < w) cp_async16(d + 16u * j, RS.src + 16u * j);
        cp_async_mbar_arrive(&c.exp_full[rs]);
        mbar_arrive(&c.exp_full[rs]);
        if (++sa == slices) {
            sa = 0;
            wk.next();
        }
        if (rs + 1 == R) rs = 0, ++round; else ++rs;
    }
    asm volatile("cp.async.wait_all;" ::: "memory");  // nothing lands after the block ends
}

template <int MAXI>
__device__ void gemm_decode(const GemmParams<MAXI>& P, const GemmSmem& S, int dw, int lane) {
    GemmCtl& c = *S.ctl;
    const uint32_t R = P.raw_stages;
    // Eight lanes per row, four rows per step, two steps per slice. Lane
    // c = lane % 8 of a row takes 16 of its 128 columns, octets o0 and o1
    // (2c, 2c+1 in the first panel; 2c+1, 2c in the second, so that the 8 lanes
    // of a row store to 8 distinct bank groups each time). Step 0 takes the
    // warp's rows 0,4,1,5 (slots 0..3), step 1 rows 2,6,3,7: the two rows of a
    // half-warp are four apart, so their exponent and mantissa loads fall in
    // complementary bank halves.
    const uint32_t c8 = uint32_t(lane) & 7u, slot = uint32_t(lane) >> 3, pp = c8 >> 2;
    const uint32_t o0 = 2u * c8 + pp, o1 = 2u * c8 + 1u - pp;
    const uint32_t row_s0 = 8u * uint32_t(dw) + (slot >> 1) + 4u * (slot & 1u), row_s1 = row_s0 + 2u;

    // slices this block works through
    uint32_t total = 0;
    {
        uint32_t it = 0;
        UnitWalk w;
        for (w.start(); w.u < P.total_units; w.next()) {
            it = find_item(P, w.u, it);
            total += P.item[it].cols / kSliceCols;
        }
    }

    uint32_t rs_g = 0, round_g = 0;  // slice g: raw stage g % R, round g / R
    for (uint32_t g = 0; g < total; ++g) {
        const uint32_t rs = rs_g, xs = g & 1u;
        const uint32_t raw_parity = round_g & 1u;
        if (rs_g + 1 == R) rs_g = 0, ++round_g; else ++rs_g;
        if (!gemm_wait_warp(&c.raw_full[rs], raw_parity, c, P.status) ||
            !gemm_wait_warp(&c.exp_full[rs], raw_parity, c, P.status) ||
            (g >= 2 && !gemm_wait_warp(&c.ax_empty[xs], ((g >> 1) - 1) & 1u, c, P.status)))
            break;
        const uint8_t* man = S.man + rs * kManStage;
        const uint8_t* exs = S.exp + rs * kExpStage;
        const uint32_t* meta = S.meta + rs * kTileRows;
        const uint32_t a_tile = smem_addr(S.a + xs * kAStage) + pp * kAPanel;
        // Every load of both steps first, the exponent words at their width-4
        // places: a step whose four rows are all of width 4 (the common case)
        // decodes from them; otherwise the step takes the general path, which
        // fetches its octets again at the rows' widths.
        uint32_t mw[2], f[2][2];
        uint4 M[2];
#pragma unroll
        for (uint32_t st = 0; st < 2; ++st) {
            const uint32_t rr = st ? row_s1 : row_s0;
            mw[st] = meta[rr];
            const uint8_t* mp = man + rr * 128u + ((c8 ^ (rr & 7u)) << 4);
            const uint2 h0 = *reinterpret_cast<const uint2*>(mp + 8u * pp);
            const uint2 h1 = *reinterpret_cast<const uint2*>(mp + 8u - 8u * pp);
            M[st] = make_uint4(h0.x, h0.y, h1.x, h1.y);
            const uint8_t* ep = exs + rr * kExpPitch;
            f[st][0] = *reinterpret_cast<const uint32_t*>(ep + 4u * o0);
            f[st][1] = *reinterpret_cast<const uint32_t*>(ep + 4u * o1);
        }
#pragma unroll
        for (uint32_t st = 0; st < 2; ++st) {
            const uint32_t rr = st ? row_s1 : row_s0;
            const uint32_t sw = rr & 7u, w = mw[st] & 0xFFu, base = mw[st] >> 8;
            uint4 v0, v1;
            if (__all_sync(0xFFFFFFFFu, w == 4u)) {
                decode_octets_w4(f[st][0], f[st][1], M[st], base * 0x00800080u, v0, v1);
            } else {
                uint4 t0, t1;
                row_constants(rr * kExpPitch, w, base, t0, t1);
                decode_octets_any(exs, t0.x + o0 * w, t0.x + o1 * w, M[st], t0, t1, v0, v1);
            }
            const uint32_t row = a_tile + rr * 128u;
            sts128(row + (((o0 & 7u) ^ sw) << 4), v0);
            sts128(row + (((o1 & 7u) ^ sw) << 4), v1);
        }
        fence_proxy_async_smem();  // the tensor cores read A through the async proxy
        __syncwarp();
        if (lane == 0) {
            mbar_arrive(&c.raw_empty[rs]);
            mbar_arrive(&c.a_full[xs]);
        }
    }
}

// ---------------------------------------------------------------------------
// MMA issue (one thread)
// ---------------------------------------------------------------------------
template <int MAXI>
__device__ void gemm_mma(const GemmParams<MAXI>& P, const GemmSmem& S) {
    GemmCtl& c = *S.ctl;
    const uint32_t idesc = bf16_idesc(kTileRows, P.nt);
    const uint32_t a0 = smem_addr(S.a), x0 = smem_addr(S.x);
    const uint32_t xstage = P.nt * 256, xpanel = P.nt * 128;
    uint32_t g = 0, j = 0, it = 0;
    bool issued = false;
    UnitWalk w;
    for (w.start(); w.u < P.total_units; w.next(), ++j) {
        it = find_item(P, w.u, it);
        const uint32_t slices = P.item[it].cols / kSliceCols;
        const uint32_t buf = j & 1u;
        if (j >= 2 && !gemm_wait(&c.acc_empty[buf], ((j >> 1) - 1) & 1u, c, P.status)) break;
        tc_fence_after();
        const uint32_t d_tmem = c.tmem_base + buf * P.nt;
        bool ok = true;
        for (uint32_t s = 0; s < slices; ++s, ++g) {
            const uint32_t xs = g & 1u;
            if (!gemm_wait(&c.a_full[xs], (g >> 1) & 1u, c, P.status) ||
                !gemm_wait(&c.x_full[xs], (g >> 1) & 1u, c, P.status)) {
                ok = false;
                break;
            }
            tc_fence_after();
            const uint32_t a = a0 + xs * kAStage, x = x0 + xs * xstage;
#pragma unroll
            for (uint32_t kk = 0; kk < kSliceCols / 16; ++kk) {
                const uint32_t off = (kk & 3u) * 32u;  // 16 BF16 = 32 bytes along K
                umma_bf16(d_tmem, sw128_desc(a + (kk >> 2) * kAPanel + off),
                          sw128_desc(x + (kk >> 2) * xpanel + off), idesc,
                          (s | kk) != 0 ? 1u : 0u);
            }
            issued = true;
            umma_commit(&c.ax_empty[xs]);
        }
        if (!ok) break;
        umma_commit(&c.acc_full[buf]);
    }
    // Every MMA has finished reading shared memory and writing TMEM before the block ends.
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
        const uint32_t buf = j & 1u;
        if (!gemm_wait_warp(&c.acc_full[buf], (j >> 1) & 1u, c, P.status, 512)) return;
        tc_fence_after();
        const uint32_t taddr = c.tmem_base + ((32u * q) << 16) + buf * P.nt;
        for (uint32_t cg = 0; cg < P.nt; cg += 16) {
            uint32_t v[16];
            tmem_ld16(taddr + cg, v);
            if (row < I.rows) {
#pragma unroll
                for (uint32_t i = 0; i < 16; ++i)
                    if (cg + i < P.tokens) I.y[uint64_t(cg + i) * I.rows + row] = __uint_as_float(v[i]);
            }
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&c.acc_empty[buf]);
    }
}

template <int MAXI>
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
    S.a = p;
    p += 2 * kAStage;
    S.x = p;
    p += 2 * P.nt * 256;
    S.man = p;
    p += P.raw_stages * kManStage;
    S.exp = p;
    p += P.raw_stages * kExpStage;
    S.meta = reinterpret_cast<uint32_t*>(p);
    GemmCtl& c = *S.ctl;
    if (tid == 0) {
        for (uint32_t s = 0; s < kMaxRawStages; ++s) {
            mbar_init(&c.raw_full[s], 1);
            mbar_init(&c.raw_empty[s], kDecWarps);
            mbar_init(&c.exp_full[s], 32 * kPrepWarps);
        }
        for (int s = 0; s < 2; ++s) {
            mbar_init(&c.a_full[s], kDecWarps);
            mbar_init(&c.x_full[s], 1);
            mbar_init(&c.ax_empty[s], 1);
            mbar_init(&c.acc_full[s], 1);
            mbar_init(&c.acc_empty[s], kEpiWarps);
        }
        mbar_init(&c.drain, 1);
        c.abort = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    if (warp == kMmaWarp) {  // tensor memory for the two accumulators
        asm volatile(
            "tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                smem_addr(&c.tmem_base)),
            "r"(P.tmem_cols)
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
    } else if (warp >= kEpiWarp0 && warp < kEpiWarp0 + kEpiWarps) {
        gemm_epilogue<MAXI>(P, S, warp, lane);
    } else if (warp == kXWarp) {
        if (lane == 0) gemm_load_x<MAXI>(P, S);
    } else if (warp >= kPrepWarp0) {
        gemm_prepare<MAXI>(P, S, warp - kPrepWarp0, lane);
    } else {
        gemm_decode<MAXI>(P, S, warp - kDecWarp0, lane);
    }

    tc_fence_before();
    __syncthreads();
    if (warp == kMmaWarp) {
        tc_fence_after();
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(c.tmem_base),
                     "r"(P.tmem_cols)
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
cudaError_t gemm_launch(const GemvItem* items, uint32_t count, uint32_t tokens, int32_t* status,
                        cudaStream_t stream) {
    static_assert(sizeof(GemmParams<MAXI>) <= 32000, "launch parameters exceed the limit");
    PFN_cuTensorMapEncodeTiled_v12000 enc = encode_fn();
    if (enc == nullptr) return cudaErrorNotSupported;
    GemmParams<MAXI> p;
    memset(&p, 0, sizeof(p));
    p.status = status;
    p.count = count;
    p.tokens = tokens;
    p.nt = (tokens + 15u) & ~15u;
    p.raw_stages = gemm_smem_bytes(p.nt, 3) <= kSmemLimit ? 3 : 2;
    p.tmem_cols = 32;
    while (p.tmem_cols < 2 * p.nt) p.tmem_cols *= 2;
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
    static uint32_t smem_set[64];
    int dev = 0;
    cudaError_t err = cudaGetDevice(&dev);
    if (err != cudaSuccess) return err;
    if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
    const uint32_t smem = gemm_smem_bytes(p.nt, p.raw_stages);
    {
        std::lock_guard<std::mutex> lock(mu);
        if (sms_of[dev] == 0) {
            err = cudaDeviceGetAttribute(&sms_of[dev], cudaDevAttrMultiProcessorCount, dev);
            if (err != cudaSuccess) return err;
        }
        if (smem_set[dev] < smem) {
            err = cudaFuncSetAttribute(gemm_kernel<MAXI>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       int(kSmemLimit));
            if (err != cudaSuccess) return err;
            smem_set[dev] = kSmemLimit;
        }
    }
    const uint64_t cap = uint64_t(sms_of[dev]);
    const unsigned grid = unsigned(units < cap ? units : cap);
    gemm_kernel<MAXI><<<grid, kGemmThreads, smem, stream>>>(p);
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_gemm(const GemvItem* items, uint32_t count, uint32_t tokens, int32_t* status,
                        cudaStream_t stream) {
    if (tokens < 1 || tokens > kMaxGemmTokens) return cudaErrorInvalidValue;
    constexpr uint32_t kBatch = kGemmBatchMax;
    if (count == 1) return gemm_launch<1>(items, 1, tokens, status, stream);
    for (uint32_t i = 0; i < count; i += kBatch) {
        const uint32_t c = min(kBatch, count - i);
        const cudaError_t err = gemm_launch<kBatch>(items + i, c, tokens, status, stream);
        if (err != cudaSuccess) return err;
    }
    return cudaSuccess;
}

}  // namespace wc
