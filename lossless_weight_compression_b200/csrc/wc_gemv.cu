// wc_gemv.cu -- fused decompression and matrix-vector products for sm_100a.
//
// y[j][r] = sum_c W[r][c] * x[j][c] for j < n_vec (1, 2 or 4), where the BF16
// weight matrix W (rows x cols, row-major) is held only as a WCB1 stream: the
// weights are decoded in shared memory and registers and never written back
// ("ZipServ: Fast and Memory-Efficient LLM Inference with Hardware-Aware
// Lossless Compression", Abstract: load compressed, compute decompressed;
// "MINE...", Abstract: single-stream decoding reads every weight once per
// token, so it is memory-bound and fewer bytes per weight is the speed-up).
//
// The kernel reuses the decoder's pipeline: a producer warp checks each tile's
// block metadata (loading the next tile's while the current one is staged) and
// bulk-copies its mantissa bytes and exponent payload into a 3-stage mbarrier
// ring; eight consumer warps decode 16 weights per chunk and accumulate
// products in FP32 with mixed-precision FMAs (BF16 x BF16 + FP32). cols must be a multiple of the block size, so every row is
// whole blocks. Work is cut into units a thread block owns whole: for
// cols <= 8192 a unit is one tile of floor(8192 / cols) rows, for wider rows a
// unit is one row, cut into tiles of up to 8192 weights. When a unit ends,
// every chunk's partial sum goes to shared memory and each row is summed over
// its chunks in a fixed order, so y is the same on every run. Waits are
// bounded by the device timer.
#include <mutex>

#include "wc_decode_core.cuh"

namespace wc {
namespace {

constexpr int kConsumerWarps = kThreads / 32;  // 8
constexpr int kProducerWarp = kConsumerWarps;
constexpr int kGemvThreads = kThreads + 32;  // 288
constexpr int kStages = 3;
constexpr int kChunksPerTile = kTile / kChunk;  // 512

template <int MAXI>
struct GemvParams {
    int32_t* status;
    uint32_t count;
    uint32_t n_vec;
    uint64_t total_units;
    uint64_t unit_begin[MAXI + 1];  // first global unit of each item; [count] = total
    uint32_t cols_magic[MAXI];      // ceil(2^32 / cols): q = umulhi(e, magic) = e / cols for e < 2^19
    GemvItem item[MAXI];
};

struct __align__(16) GemvInfo {
    const uint16_t* x;  // x of this item, at this tile's first column
    float* y;           // y of this item, at the unit's first row
    uint32_t len;       // weights to decode in this tile (0: corrupt tile, skip)
    uint32_t log2B;
    uint32_t cols;      // row length and stride between the x vectors
    uint32_t rows;      // stride between the y vectors
    uint32_t magic;     // ceil(2^32 / cols)
    uint32_t nrows;     // rows of the unit (0: no more work)
    uint32_t last;      // last tile of its unit: reduce and write y
    uint32_t pad[3];
};

struct __align__(16) GemvStage {
    uint8_t man[kTile];
    uint8_t exp[kTile + 16];
    uint4 t0[kMaxBlocksPerTile];
    uint4 t1[kMaxBlocksPerTile];
    GemvInfo info;
};

template <int NV>
struct GemvSmem {
    GemvStage stage[kStages];
    unsigned long long full[kStages], empty[kStages];
    unsigned long long unit_done[2];            // the 8 consumer warps, by unit parity
    float part[2][kChunksPerTile][NV];          // per-chunk partial sums, by unit parity
    int abort;
};

template <int MAXI>
__device__ __forceinline__ uint32_t find_item(const GemvParams<MAXI>& P, uint64_t u, uint32_t from) {
    while (u >= P.unit_begin[from + 1]) ++from;
    return from;
}

// Geometry of unit u_local of an item: its first row, rows and tiles.
__device__ __forceinline__ void unit_geometry(const GemvItem& I, uint64_t u_local,
                                              uint64_t& first_row, uint32_t& nrows,
                                              uint32_t& ntiles) {
    if (I.cols <= uint32_t(kTile)) {
        const uint32_t per = uint32_t(kTile) / I.cols;
        first_row = u_local * per;
        nrows = uint32_t(min(uint64_t(per), uint64_t(I.rows) - first_row));
        ntiles = 1;
    } else {
        first_row = u_local;
        nrows = 1;
        ntiles = (I.cols + kTile - 1) / kTile;
    }
}

// Tile j of a unit: first weight and weight count.
__device__ __forceinline__ void tile_geometry(const GemvItem& I, uint64_t first_row, uint32_t nrows,
                                              uint32_t j, uint64_t& first, uint32_t& len) {
    if (I.cols <= uint32_t(kTile)) {
        first = first_row * I.cols;
        len = nrows * I.cols;
    } else {
        first = first_row * I.cols + uint64_t(j) * kTile;
        len = min(uint32_t(kTile), I.cols - j * uint32_t(kTile));
    }
}

template <int NV>
__device__ __forceinline__ void give_up(GemvSmem<NV>& sm, int32_t* status, int lane) {
    if (lane == 0) {
        report(status, kStatusTimeout);
        sm.abort = 1;
    }
}

// ---------------------------------------------------------------------------
// producer warp: units blockIdx.x, blockIdx.x + gridDim.x, ..., tile by tile
// ---------------------------------------------------------------------------
template <int MAXI, int NV>
__device__ void gemv_produce(const GemvParams<MAXI>& P, GemvSmem<NV>& sm, int lane) {
    // the current tile, and the next one whose metadata is already on its way
    struct Cur {
        uint64_t u, first_row, first;
        uint32_t it, nrows, ntiles, j, len;
        bool valid;
    };
    auto locate = [&](uint64_t u, uint32_t j, uint32_t from) {
        Cur c = {};
        c.u = u;
        c.j = j;
        c.valid = u < P.total_units;
        if (!c.valid) return c;
        c.it = find_item(P, u, from);
        const GemvItem& I = P.item[c.it];
        unit_geometry(I, u - P.unit_begin[c.it], c.first_row, c.nrows, c.ntiles);
        tile_geometry(I, c.first_row, c.nrows, j, c.first, c.len);
        return c;
    };
    auto advance = [&](const Cur& c) {
        return c.j + 1 < c.ntiles ? locate(c.u, c.j + 1, c.it) : locate(c.u + gridDim.x, 0, c.it);
    };
    auto load_meta = [&](const Cur& c) {
        TileMeta m = {};
        if (c.valid) {
            const GemvItem& I = P.item[c.it];
            m = load_tile_meta(I.stream, make_layout(uint64_t(I.rows) * I.cols, I.block), c.first,
                               c.len, lane);
        }
        return m;
    };
    int issued_round[kStages];
    for (int s = 0; s < kStages; ++s) issued_round[s] = -1;
    Cur cur = locate(blockIdx.x, 0, 0);
    TileMeta meta = load_meta(cur);
    for (uint32_t i = 0;; ++i) {
        const Cur next = cur.valid ? advance(cur) : cur;
        const TileMeta meta_next = load_meta(next);
        const int s = int(i % kStages);
        const uint32_t round = i / kStages;
        if (round > 0 && !mbar_wait(&sm.empty[s], (round & 1u) ^ 1u, &sm.abort, 256)) {
            give_up(sm, P.status, lane);
            if (lane == 0)
                for (int k = 0; k < kStages; ++k)
                    if (issued_round[k] >= 0)
                        mbar_wait(&sm.full[k], uint32_t(issued_round[k]) & 1u, nullptr);
            return;
        }
        GemvStage& st = sm.stage[s];
        if (!cur.valid) {  // no more units: tell the consumers
            if (lane == 0) {
                st.info.nrows = 0;
                mbar_arrive(&sm.full[s]);
            }
            return;
        }
        const GemvItem& I = P.item[cur.it];
        const Layout L = make_layout(uint64_t(I.rows) * I.cols, I.block);
        if (cur.first == 0 && lane == 0) {
            DecodeItem d;
            d.stream = I.stream;
            d.stream_bytes = I.stream_bytes;
            check_container(d, L, P.status);
        }
        uint64_t start = 0;
        uint32_t len16 = 0;
        const bool ok = commit_tile_meta(meta, I.stream, L, I.stream_bytes, cur.len, st.t0, st.t1,
                                         st.exp, start, len16, lane);
        if (!ok && lane == 0) report(P.status, kStatusCorrupt);
        if (lane == 0) {
            const uint64_t col0 = I.cols <= uint32_t(kTile) ? 0 : uint64_t(cur.j) * kTile;
            st.info = GemvInfo{I.x + col0, I.y + cur.first_row, ok ? cur.len : 0u, L.log2_block,
                               I.cols, I.rows, P.cols_magic[cur.it], cur.nrows,
                               cur.j + 1 == cur.ntiles ? 1u : 0u, {0u, 0u, 0u}};
        }
        __syncwarp();
        if (lane == 0) {
            if (!ok) {
                mbar_arrive(&sm.full[s]);
            } else {
                mbar_arrive_expect_tx(&sm.full[s], cur.len + len16);  // len: a multiple of 128
                bulk_load(st.man, I.stream + L.off_man + cur.first, cur.len, &sm.full[s]);
                if (len16) bulk_load(st.exp, I.stream + L.off_exp + start, len16, &sm.full[s]);
                issued_round[s] = int(round);
            }
        }
        cur = next;
        meta = meta_next;
    }
}

// ---------------------------------------------------------------------------
// consumer warps
// ---------------------------------------------------------------------------
// acc + a * b for two BF16 values and an FP32 accumulator, one rounding (the
// product of two BF16 values is exact in FP32).
__device__ __forceinline__ float fma_bf16(uint32_t a, uint32_t b, float acc) {
    float d;
    asm("fma.rn.f32.bf16 %0, %1, %2, %3;" : "=f"(d) : "h"(uint16_t(a)), "h"(uint16_t(b)), "f"(acc));
    return d;
}

// acc + sum over 8 weights (4 BF16 pairs in w) times 8 x values (4 pairs in v),
// in element order.
__device__ __forceinline__ float dot8(uint4 w, uint4 v, float acc) {
    acc = fma_bf16(w.x, v.x, acc);
    acc = fma_bf16(w.x >> 16, v.x >> 16, acc);
    acc = fma_bf16(w.y, v.y, acc);
    acc = fma_bf16(w.y >> 16, v.y >> 16, acc);
    acc = fma_bf16(w.z, v.z, acc);
    acc = fma_bf16(w.z >> 16, v.z >> 16, acc);
    acc = fma_bf16(w.w, v.w, acc);
    acc = fma_bf16(w.w >> 16, v.w >> 16, acc);
    return acc;
}

__device__ __forceinline__ uint4 ld_x(const uint16_t* p) {
    uint4 v;
    asm volatile("ld.global.nc.v4.u32 {%0,%1,%2,%3}, [%4];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                 : "l"(p));
    return v;
}

template <int NV>
__device__ void gemv_consume(GemvSmem<NV>& sm, int32_t* status, int tid, int lane, int warp) {
    float acc[kChunksPerThread][NV];
#pragma unroll
    for (int k = 0; k < kChunksPerThread; ++k)
#pragma unroll
        for (int j = 0; j < NV; ++j) acc[k][j] = 0.f;
    uint32_t units = 0;
    for (uint32_t i = 0;; ++i) {
        const int s = int(i % kStages);
        const uint32_t round = i / kStages;
        if (!mbar_wait(&sm.full[s], round & 1u, &sm.abort)) {
            give_up(sm, status, lane);
            return;
        }
        const GemvStage& st = sm.stage[s];
        const GemvInfo info = st.info;
        if (info.nrows == 0) return;
        const uint32_t bmask = (1u << info.log2B) - 1u;
#pragma unroll
        for (int k = 0; k < kChunksPerThread; ++k) {
            const uint32_t el = uint32_t(tid + k * kThreads) * kChunk;
            if (el >= info.len) continue;
            const uint4 M = *reinterpret_cast<const uint4*>(st.man + el);
            const uint4 t0 = st.t0[el >> info.log2B], t1 = st.t1[el >> info.log2B];
            const uint32_t q = t0.x + ((el & bmask) >> 3) * t0.y;
            uint4 w0, w1;
            decode_chunk(st.exp, q, M, t0, t1, w0, w1);
            const uint32_t row = __umulhi(el, info.magic);  // el / cols
            const uint32_t col = el - row * info.cols;
#pragma unroll
            for (int j = 0; j < NV; ++j) {
                const uint16_t* xp = info.x + uint64_t(j) * info.cols + col;
                acc[k][j] = dot8(w1, ld_x(xp + 8), dot8(w0, ld_x(xp), acc[k][j]));
            }
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&sm.empty[s]);
        if (!info.last) continue;

        // ---- the unit is complete: chunk partials to shared memory, rows summed in order
        const int buf = int(units & 1u);
#pragma unroll
        for (int k = 0; k < kChunksPerThread; ++k)
#pragma unroll
            for (int j = 0; j < NV; ++j) {
                sm.part[buf][tid + k * kThreads][j] = acc[k][j];
                acc[k][j] = 0.f;
            }
        __syncwarp();
        if (lane == 0) mbar_arrive(&sm.unit_done[buf]);
        if (!mbar_wait(&sm.unit_done[buf], (units >> 1) & 1u, &sm.abort)) {
            give_up(sm, status, lane);
            return;
        }
        const uint32_t per_row = min(info.cols, uint32_t(kTile)) / kChunk;  // chunks of a row
        for (uint32_t r = warp; r < info.nrows; r += kConsumerWarps) {
#pragma unroll
            for (int j = 0; j < NV; ++j) {
                float v = 0.f;
                for (uint32_t c = lane; c < per_row; c += 32) v += sm.part[buf][r * per_row + c][j];
#pragma unroll
                for (int off = 16; off > 0; off >>= 1) v += __shfl_xor_sync(0xFFFFFFFFu, v, off);
                if (lane == 0) info.y[uint64_t(j) * info.rows + r] = v;
            }
        }
        ++units;
    }
}

template <int MAXI, int NV>
__global__ void __launch_bounds__(kGemvThreads)
    gemv_kernel(const __grid_constant__ GemvParams<MAXI> P) {
    extern __shared__ __align__(128) unsigned char smem_raw[];
    GemvSmem<NV>& sm = *reinterpret_cast<GemvSmem<NV>*>(smem_raw);
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    if (tid == 0) {
        for (int s = 0; s < kStages; ++s) {
            mbar_init(&sm.full[s], 1);
            mbar_init(&sm.empty[s], kConsumerWarps);
        }
        mbar_init(&sm.unit_done[0], kConsumerWarps);
        mbar_init(&sm.unit_done[1], kConsumerWarps);
        sm.abort = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    __syncthreads();
    if (warp == kProducerWarp)
        gemv_produce<MAXI, NV>(P, sm, lane);
    else
        gemv_consume<NV>(sm, P.status, tid, lane, warp);
}

template <int MAXI, int NV>
cudaError_t gemv_grid(uint64_t units, unsigned* grid) {
    static std::mutex mu;
    static int per_device[64];
    int dev = 0;
    cudaError_t err = cudaGetDevice(&dev);
    if (err != cudaSuccess) return err;
    if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
    std::lock_guard<std::mutex> lock(mu);
    if (per_device[dev] == 0) {
        err = cudaFuncSetAttribute(gemv_kernel<MAXI, NV>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                   int(sizeof(GemvSmem<NV>)));
        if (err != cudaSuccess) return err;
        int sms = 0, per_sm = 0;
        err = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
        if (err != cudaSuccess) return err;
        err = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, gemv_kernel<MAXI, NV>,
                                                            kGemvThreads, sizeof(GemvSmem<NV>));
        if (err != cudaSuccess) return err;
        per_device[dev] = (per_sm > 0 ? per_sm : 1) * sms;
    }
    const uint64_t cap = uint64_t(per_device[dev]);
    *grid = unsigned(units < cap ? units : cap);
    return cudaSuccess;
}

uint64_t units_of(const GemvItem& I) {
    if (I.rows == 0) return 0;
    if (I.cols <= uint32_t(kTile)) {
        const uint32_t per = uint32_t(kTile) / I.cols;
        return (uint64_t(I.rows) + per - 1) / per;
    }
    return I.rows;
}

template <int MAXI, int NV>
cudaError_t gemv_batch(const GemvItem* items, uint32_t count, int32_t* status,
                       cudaStream_t stream) {
    static_assert(sizeof(GemvParams<MAXI>) <= 32000, "launch parameters exceed the limit");
    GemvParams<MAXI> p;
    p.status = status;
    p.count = count;
    p.n_vec = NV;
    uint64_t units = 0;
    for (uint32_t i = 0; i < count; ++i) {
        p.unit_begin[i] = units;
        p.item[i] = items[i];
        p.cols_magic[i] = uint32_t((0x100000000ull + items[i].cols - 1) / items[i].cols);
        units += units_of(items[i]);
    }
    p.unit_begin[count] = units;
    p.total_units = units;
    if (units == 0) return cudaSuccess;
    unsigned grid = 0;
    cudaError_t err = gemv_grid<MAXI, NV>(units, &grid);
    if (err != cudaSuccess) return err;
    gemv_kernel<MAXI, NV><<<grid, kGemvThreads, sizeof(GemvSmem<NV>), stream>>>(p);
    return cudaGetLastError();
}

template <int NV>
cudaError_t gemv_nv(const GemvItem* items, uint32_t count, int32_t* status, cudaStream_t stream) {
    constexpr uint32_t kBatch = 256;
    if (count == 1) return gemv_batch<1, NV>(items, 1, status, stream);
    for (uint32_t i = 0; i < count; i += kBatch) {
        const uint32_t c = min(kBatch, count - i);
        const cudaError_t err = gemv_batch<kBatch, NV>(items + i, c, status, stream);
        if (err != cudaSuccess) return err;
    }
    return cudaSuccess;
}

}  // namespace

cudaError_t launch_gemv(const GemvItem* items, uint32_t count, uint32_t n_vec, int32_t* status,
                        cudaStream_t stream) {
    switch (n_vec) {
        case 1: return gemv_nv<1>(items, count, status, stream);
        case 2: return gemv_nv<2>(items, count, status, stream);
        case 4: return gemv_nv<4>(items, count, status, stream);
        default: return cudaErrorInvalidValue;
    }
}

}  // namespace wc
