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
//   - a producer warp reads each slice's per-row block headers and offsets,
//     checks them, and starts the copies: the slice's mantissa bytes (one 2-D
//     TMA load, 128-byte swizzled), each row's exponent bytes (one bulk copy per
//     row; a 128-column slice of a row is 16 whole octets of one block, 16*w
//     bytes), and the activations (two 2-D TMA loads, 128-byte swizzled, which
//     is the K-major layout the MMA reads);
//   - eight decoding warps turn the staged bytes into BF16 weights and store
//     them in the same K-major 128-byte-swizzled layout;
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

#include <mutex>

#include "wc_decode_core.cuh"

namespace wc {
namespace {

constexpr uint32_t kTileRows = 128;    // MMA M
constexpr uint32_t kSliceCols = 128;   // columns per pipeline slice (8 MMAs of K = 16)
constexpr uint32_t kExpPitch = 144;    // staged exponent bytes per row (16*w <= 128, +16 spreads banks)
constexpr uint32_t kManStage = kTileRows * kSliceCols;      // 16 KB
constexpr uint32_t kExpStage = kTileRows * kExpPitch;       // 18 KB
constexpr uint32_t kMetaStage = kTileRows * 2 * 16;         // t0 and t1 per row
constexpr uint32_t kAStage = kTileRows * kSliceCols * 2;    // 32 KB: two 64-column panels
constexpr uint32_t kAPanel = kTileRows * 128;               // 128 rows x 128 bytes
constexpr uint32_t kMaxRawStages = 3;
constexpr uint32_t kSmemLimit = 232448;                     // 227 KB per block

constexpr int kProducerWarp = 0;
constexpr int kMmaWarp = 1;
constexpr int kEpiWarp0 = 2;   // warps 2..5: warp % 4 covers the four TMEM lane quarters
constexpr int kEpiWarps = 4;
constexpr int kDecWarp0 = 6;
constexpr int kDecWarps = 8;
constexpr int kGemmThreads = 32 * (kDecWarp0 + kDecWarps);  // 448
constexpr int kChunksPerDecThread = int(kSliceCols / 16) * 4 / kDecWarps;  // 4

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
    uint4* meta;    // per stage: t0[128], t1[128]
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
// producer warp
// ---------------------------------------------------------------------------
template <int MAXI>
__device__ void gemm_produce(const GemmParams<MAXI>& P, const GemmSmem& S, int lane) {
    GemmCtl& c = *S.ctl;
    const uint32_t R = P.raw_stages;
    uint32_t g = 0, it = 0;
    // phases this warp started on each barrier, to drain them if the block stops early
    int raw_issued[kMaxRawStages] = {-1, -1, -1};
    int x_issued[2] = {-1, -1};
    bool ok = true;
    for (uint64_t u = blockIdx.x; ok && u < P.total_units; u += gridDim.x) {
        it = find_item(P, u, it);
        const GemvItem& I = P.item[it];
        const uint64_t n = uint64_t(I.rows) * I.cols;
        const Layout L = make_layout(n, I.block);
        const uint8_t* St = I.stream;
        const uint32_t row0 = uint32_t(u - P.unit_begin[it]) * kTileRows;
        if (row0 == 0 && lane == 0) {
            DecodeItem d;
            d.stream = St;
            d.stream_bytes = I.stream_bytes;
            check_container(d, L, P.status);
        }
        const uint16_t* hdr = reinterpret_cast<const uint16_t*>(St + L.off_hdr);
        const uint32_t* offs = reinterpret_cast<const uint32_t*>(St + L.off_offs);
        const uint32_t bmask = L.block - 1u;
        const uint32_t slices = I.cols / kSliceCols;
        for (uint32_t s = 0; s < slices; ++s, ++g) {
            const uint32_t k0 = s * kSliceCols;
            // 1. this lane's rows' block headers and offsets (loaded before the wait)
            uint32_t h[4];
            uint64_t sb[4], nx[4], el[4];
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                const uint32_t r = uint32_t(lane) + 32u * j;
                h[j] = 0;
                sb[j] = nx[j] = 0;
                el[j] = 0;
                if (row0 + r < I.rows) {
                    el[j] = uint64_t(row0 + r) * I.cols + k0;
                    const uint64_t b = el[j] >> L.log2_block;
                    h[j] = hdr[b];
                    sb[j] = 16ull * offs[b];
                    if ((el[j] & bmask) == 0)  // first slice of the block: check the offset chain
                        nx[j] = b + 1 < L.nb ? 16ull * offs[b + 1] : ld_u64(St + 64);
                }
            }
            // 2. a free raw stage
            const uint32_t rs = g % R;
            if (g >= R && !gemm_wait_warp(&c.raw_empty[rs], ((g / R) - 1) & 1u, c, P.status, 256)) {
                ok = false;
                break;
            }
            uint8_t* man = S.man + rs * kManStage;
            uint8_t* exs = S.exp + rs * kExpStage;
            uint4* t0 = S.meta + rs * 2 * kTileRows;
            uint4* t1 = t0 + kTileRows;
            // 3. check, write the decode constants, size the copies
            uint32_t bytes[4];
            uint64_t src[4];
            uint32_t total = 0;
            bool bad = false;
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                const uint32_t r = uint32_t(lane) + 32u * j;
                uint32_t w = h[j] >> 8, base = h[j] & 0xFFu;
                bytes[j] = 0;
                src[j] = 0;
                if (row0 + r < I.rows) {
                    bool b_bad = w > 8u || (w == 8u && base != 0u);
                    if ((el[j] & bmask) == 0) {
                        const uint64_t blk = el[j] >> L.log2_block;
                        const uint64_t len = min(uint64_t(L.block), n - (blk << L.log2_block));
                        b_bad |= sb[j] + ((len + 7) >> 3) * min(w, 8u) != nx[j];
                    }
                    const uint64_t seg = (el[j] & bmask) >> 3;  // first octet of the slice
                    src[j] = L.off_exp + sb[j] + seg * min(w, 8u);
                    b_bad |= src[j] + 16ull * min(w, 8u) > I.stream_bytes;
                    if (b_bad) {
                        bad = true;
                        w = 0;
                        base = 0;
                    }
                    bytes[j] = 16u * w;
                } else {
                    w = 0;
                    base = 0;
                }
                const uint32_t m1 = (1u << w) - 1u;
                t0[r] = make_uint4(r * kExpPitch, w, 2 * w, 4 * w);
                t1[r] = make_uint4(m1 | (m1 << 16), (1u << (2 * w)) - 1u,
                                   w == 8u ? 0xFFFFFFFFu : (1u << (4 * w)) - 1u,
                                   base * 0x00800080u);
                total += bytes[j];
            }
            if (__any_sync(0xFFFFFFFFu, bad) && lane == 0) report(P.status, kStatusCorrupt);
            total = __reduce_add_sync(0xFFFFFFFFu, total) + kManStage;
            __syncwarp();
            if (lane == 0) {
                mbar_arrive_expect_tx(&c.raw_full[rs], total);
                tma_load_2d(man, &P.man_map[it], int32_t(k0), int32_t(row0), &c.raw_full[rs]);
                raw_issued[rs] = int(g / R);
            }
            __syncwarp();
#pragma unroll
            for (int j = 0; j < 4; ++j)
                if (bytes[j])
                    bulk_load(exs + (uint32_t(lane) + 32u * j) * kExpPitch, St + src[j], bytes[j],
                              &c.raw_full[rs]);
            // 4. a free activation stage (the MMAs of slice g - 2 are done)
            const uint32_t xs = g & 1u;
            if (g >= 2 && !gemm_wait_warp(&c.ax_empty[xs], ((g >> 1) - 1) & 1u, c, P.status, 256)) {
                ok = false;
                break;
            }
            if (lane == 0) {
                uint8_t* xd = S.x + xs * P.nt * 256;
                mbar_arrive_expect_tx(&c.x_full[xs], P.nt * 256);
                tma_load_2d(xd, &P.x_map[it], int32_t(k0), 0, &c.x_full[xs]);
                tma_load_2d(xd + P.nt * 128, &P.x_map[it], int32_t(k0 + 64), 0, &c.x_full[xs]);
                x_issued[xs] = int(g >> 1);
            }
        }
    }
    // Stopped early: let the copies already started land before the block exits.
    if (!ok && lane == 0) {
        for (uint32_t k = 0; k < R; ++k)
            if (raw_issued[k] >= 0) mbar_wait(&c.raw_full[k], uint32_t(raw_issued[k]) & 1u, nullptr);
        for (int k = 0; k < 2; ++k)
            if (x_issued[k] >= 0) mbar_wait(&c.x_full[k], uint32_t(x_issued[k]) & 1u, nullptr);
    }
}

// ---------------------------------------------------------------------------
// decoding warps: warp d decodes rows 32*(d%4) .. +31, chunks 4*(d/4) .. +3 of
// every slice (a chunk is 16 columns). A lane owns one row, so each of its
// chunks is one 16-byte swizzled mantissa load, 2w exponent bytes, and two
// 16-byte swizzled stores; the 32 lanes of a warp hit 32 different rows, which
// the swizzle spreads over all banks.
// ---------------------------------------------------------------------------
template <int MAXI>
__device__ void gemm_decode(const GemmParams<MAXI>& P, const GemmSmem& S, int dw, int lane) {
    GemmCtl& c = *S.ctl;
    const uint32_t R = P.raw_stages;
    const uint32_t r = 32u * (dw & 3) + uint32_t(lane);
    const uint32_t c0 = uint32_t(dw >> 2) * kChunksPerDecThread;
    const uint32_t sw = r & 7u;
    uint32_t g = 0, it = 0;
    for (uint64_t u = blockIdx.x; u < P.total_units; u += gridDim.x) {
        it = find_item(P, u, it);
        const uint32_t slices = P.item[it].cols / kSliceCols;
        for (uint32_t s = 0; s < slices; ++s, ++g) {
            const uint32_t rs = g % R, xs = g & 1u;
            if (!gemm_wait_warp(&c.raw_full[rs], (g / R) & 1u, c, P.status)) return;
            if (g >= 2 && !gemm_wait_warp(&c.ax_empty[xs], ((g >> 1) - 1) & 1u, c, P.status)) return;
            const uint8_t* man = S.man + rs * kManStage + r * 128u;
            const uint8_t* exs = S.exp + rs * kExpStage;
            const uint4* meta = S.meta + rs * 2 * kTileRows;
            const uint4 t0 = meta[r], t1 = meta[kTileRows + r];
            const uint32_t a_row = smem_addr(S.a + xs * kAStage) + r * 128u;
#pragma unroll
            for (int i = 0; i < kChunksPerDecThread; ++i) {
                const uint32_t ch = c0 + uint32_t(i);
                const uint4 M = *reinterpret_cast<const uint4*>(man + (((ch & 7u) ^ sw) << 4));
                uint4 v0, v1;
                decode_chunk(exs, t0.x + ch * t0.z, M, t0, t1, v0, v1);
                const uint32_t panel = a_row + (ch >> 2) * kAPanel;
                const uint32_t j0 = (ch & 3u) * 2u;
                sts128(panel + ((j0 ^ sw) << 4), v0);
                sts128(panel + (((j0 + 1u) ^ sw) << 4), v1);
            }
            fence_proxy_async_smem();  // the tensor cores read A through the async proxy
            __syncwarp();
            if (lane == 0) {
                mbar_arrive(&c.raw_empty[rs]);
                mbar_arrive(&c.a_full[xs]);
            }
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
    for (uint64_t u = blockIdx.x; u < P.total_units; u += gridDim.x, ++j) {
        it = find_item(P, u, it);
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
    for (uint64_t u = blockIdx.x; u < P.total_units; u += gridDim.x, ++j) {
        it = find_item(P, u, it);
        const GemvItem& I = P.item[it];
        const uint32_t row = uint32_t(u - P.unit_begin[it]) * kTileRows + 32u * q + uint32_t(lane);
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
    S.meta = reinterpret_cast<uint4*>(p);
    GemmCtl& c = *S.ctl;
    if (tid == 0) {
        for (uint32_t s = 0; s < kMaxRawStages; ++s) {
            mbar_init(&c.raw_full[s], 1);
            mbar_init(&c.raw_empty[s], kDecWarps);
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
        gemm_produce<MAXI>(P, S, lane);
    } else if (warp == kMmaWarp) {
        if (lane == 0) gemm_mma<MAXI>(P, S);
    } else if (warp >= kEpiWarp0 && warp < kEpiWarp0 + kEpiWarps) {
        gemm_epilogue<MAXI>(P, S, warp, lane);
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
    uint64_t units = 0;
    for (uint32_t i = 0; i < count; ++i) {
        const GemvItem& I = items[i];
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
