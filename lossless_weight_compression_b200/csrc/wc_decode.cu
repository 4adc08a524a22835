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
// One thread block decodes one 8192-element tile of one tensor:
//   1. 16-byte loads of the tile's mantissa bytes are issued first (their
//      address depends on nothing in the stream);
//   2. the tile's block headers and offsets are read and checked (w <= 8,
//      base 0 when raw, offsets equal to the prefix sum of the block sizes,
//      every byte inside the stream);
//   3. the tile's exponent payload -- contiguous, starting 16-byte aligned --
//      is staged in shared memory with 16-byte loads;
//   4. each thread unpacks two octets per 16-element chunk by reversing the
//      hierarchical halving (octet -> quads -> pairs -> values), adds the
//      base, merges sign and mantissa, and writes 32 bytes of BF16 with
//      16-byte stores.
// A batch of tensors is one launch: the per-tensor descriptors travel as
// launch parameters, and each thread block finds its tensor by a binary search
// over the tensors' first tile indices.
#include "wc_internal.cuh"

namespace wc {
namespace {

template <int MAXI>
struct DecodeParams {
    int32_t* status;
    uint32_t count;
    uint32_t pad;
    uint64_t tile_begin[MAXI + 1];  // first global tile of each item; [count] = total
    DecodeItem item[MAXI];
};

// Eight w-bit values of one octet (lo/hi = its 64 bits; bits above 8w are
// ignored) -> four words, each holding two finished BF16 values.
//   quads: q0 = bits [0,4w), q1 = bits [4w,8w)
//   pairs: p0 = q0 & m2, p1 = q0 >> 2w (taken from lo:hi), p2 = q1 & m2, p3 = q1 >> 2w
//   pair -> two 16-bit lanes: (p & m1) | (p >> w & m1) << 16
//   lane  -> BF16:  (v + base) << 7 | sign << 15 | mantissa
struct OctetDecoder {
    uint32_t w, m1, m1_hi, m2, m4, base7;
    __device__ __forceinline__ OctetDecoder(uint32_t w_, uint32_t base) {
        w = w_;
        m1 = (1u << w) - 1u;
        m1_hi = m1 << 16;
        m2 = (1u << (2 * w)) - 1u;
        m4 = (w == 8u) ? 0xFFFFFFFFu : ((1u << (4 * w)) - 1u);
        base7 = base * 0x00800080u;  // base at bit 7 of both 16-bit lanes
    }
    __device__ __forceinline__ uint32_t lanes(uint32_t pair) const {
        const uint32_t v = (pair & m1) | ((pair << (16 - w)) & m1_hi);
        return v * 128u + base7;  // exponent field of both lanes: (v + base) << 7
    }
    // s4: the four sign+mantissa bytes of elements 0..3 (first) or 4..7
    __device__ __forceinline__ uint4 decode(uint32_t lo, uint32_t hi, uint32_t s_lo4,
                                            uint32_t s_hi4) const {
        const uint32_t p0 = lo & m2;
        const uint32_t p1 = __funnelshift_r(lo, hi, 2 * w) & m2;
        const uint32_t q1 = __funnelshift_rc(lo, hi, 4 * w) & m4;
        const uint32_t p2 = q1 & m2;
        const uint32_t p3 = q1 >> (2 * w);
        // sign+mantissa byte s replicated into both bytes of a lane: & 0x807F
        // keeps the mantissa in bits 0..6 and moves the sign to bit 15.
        uint4 r;
        r.x = (prmt(s_lo4, 0u, 0x1100u) & 0x807F807Fu) | lanes(p0);
        r.y = (prmt(s_lo4, 0u, 0x3322u) & 0x807F807Fu) | lanes(p1);
        r.z = (prmt(s_hi4, 0u, 0x1100u) & 0x807F807Fu) | lanes(p2);
        r.w = (prmt(s_hi4, 0u, 0x3322u) & 0x807F807Fu) | lanes(p3);
        return r;
    }
};

// 64 bits starting at byte q of the staged exponent bytes (q need not be aligned).
__device__ __forceinline__ void fetch_octet(const uint32_t* s32, uint32_t q, uint32_t& lo,
                                            uint32_t& hi) {
    const uint32_t a = q >> 2, r = (q & 3u) * 8u;
    const uint32_t x0 = s32[a], x1 = s32[a + 1], x2 = s32[a + 2];
    lo = __funnelshift_r(x0, x1, r);
    hi = __funnelshift_r(x1, x2, r);
}

__device__ __forceinline__ uint64_t ld_u64(const uint8_t* p) {
    return *reinterpret_cast<const uint64_t*>(p);
}

// Thread block 0 of each tensor checks the container header against (n, B).
__device__ void check_container(const DecodeItem& I, const Layout& L, int32_t* status) {
    const uint8_t* S = I.stream;
    bool bad = ld_u64(S) != (kMagic | (uint64_t(kVersion) << 32) | (uint64_t(kHeaderBytes) << 48));
    bad |= ld_u64(S + 8) != uint64_t(L.block);  // block size, flags = 0
    bad |= ld_u64(S + 16) != L.n;
    bad |= ld_u64(S + 24) != L.nb;
    bad |= ld_u64(S + 32) != L.off_hdr;
    bad |= ld_u64(S + 40) != L.off_offs;
    bad |= ld_u64(S + 48) != L.off_man;
    bad |= ld_u64(S + 56) != L.off_exp;
    const uint64_t E = ld_u64(S + 64), total = ld_u64(S + 72);
    bad |= E > L.n + 8 || total != L.off_exp + E || total > I.stream_bytes;
    for (int k = 80; k < 128; k += 8) bad |= ld_u64(S + k) != 0;
    if (bad) report(status, kStatusCorrupt);
}

template <int MAXI>
__global__ void __launch_bounds__(kThreads) decode_kernel(const __grid_constant__ DecodeParams<MAXI> P) {
    __shared__ __align__(16) uint8_t s_exp[kTile + 16];
    __shared__ uint32_t s_hdr[kMaxBlocksPerTile];
    __shared__ uint32_t s_off[kMaxBlocksPerTile];
    __shared__ uint32_t s_blk[kMaxBlocksPerTile];  // base | w << 8 | staged byte offset << 16
    __shared__ unsigned long long s_next, s_start;
    __shared__ uint32_t s_len;
    __shared__ int s_bad;

    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const uint64_t gt = blockIdx.x;

    int it = 0;
    if (MAXI > 1) {  // the last item whose first tile is <= gt
        int lo = 0, hi = int(P.count) - 1;
        while (lo < hi) {
            const int mid = (lo + hi + 1) >> 1;
            if (P.tile_begin[mid] <= gt) lo = mid; else hi = mid - 1;
        }
        it = lo;
    }
    const DecodeItem& I = P.item[it];
    const uint64_t lt = gt - P.tile_begin[it];
    const Layout L = make_layout(I.n, I.block);
    const uint8_t* S = I.stream;

    if (lt == 0 && tid == 32) check_container(I, L, P.status);
    if (L.n == 0) return;  // an empty tensor's tile only checks the header

    const uint32_t log2B = L.log2_block, B = L.block;
    const uint64_t tile_start = lt * kTile;
    const uint32_t tile_n = uint32_t(min(uint64_t(kTile), L.n - tile_start));
    const uint64_t b0 = tile_start >> log2B;
    const uint32_t nblk = (tile_n + B - 1) >> log2B;

    // 1. mantissa bytes (the mantissa section is padded to 128 bytes and the
    //    host checked stream_bytes >= off_exp, so full 16-byte loads stay inside)
    uint4 M[kChunksPerThread];
#pragma unroll
    for (int k = 0; k < kChunksPerThread; ++k) {
        const uint32_t el = uint32_t(tid + k * kThreads) * kChunk;
        if (el < tile_n) M[k] = ld_stream_v4(S + L.off_man + tile_start + el);
    }
    // 2. block headers and offsets of the tile, and where the next tile starts
    if (tid < nblk) {
        s_hdr[tid] = reinterpret_cast<const uint16_t*>(S + L.off_hdr)[b0 + tid];
        s_off[tid] = reinterpret_cast<const uint32_t*>(S + L.off_offs)[b0 + tid];
    } else if (tid == nblk) {
        s_next = (b0 + nblk < L.nb) ? 16ull * reinterpret_cast<const uint32_t*>(S + L.off_offs)[b0 + nblk]
                                    : ld_u64(S + 64);  // after the last block: E
    }
    __syncthreads();
    if (warp == 0) {
        bool bad = false;
        unsigned long long start_j[2];
        uint32_t blk[2];
#pragma unroll
        for (int j = 0; j < 2; ++j) {
            const uint32_t i = 2 * lane + j;
            start_j[j] = 0;
            blk[j] = 0;
            if (i < nblk) {
                const uint32_t h = s_hdr[i], w = h >> 8, base = h & 0xFFu;
                bad |= w > 8u || (w == 8u && base != 0u);
                const uint32_t len = min(B, tile_n - i * B);
                const uint64_t size = uint64_t((len + 7) >> 3) * min(w, 8u);
                start_j[j] = 16ull * s_off[i];
                const uint64_t next = (i + 1 < nblk) ? 16ull * s_off[i + 1] : s_next;
                bad |= start_j[j] + size != next;
                blk[j] = h;
            }
        }
        const unsigned long long start = 16ull * s_off[0], end = s_next;
        bad |= end > I.stream_bytes - L.off_exp;
        bad = __any_sync(0xFFFFFFFFu, bad);
#pragma unroll
        for (int j = 0; j < 2; ++j) {
            const uint32_t i = 2 * lane + j;
            if (i < nblk && !bad) s_blk[i] = blk[j] | (uint32_t(start_j[j] - start) << 16);
        }
        if (lane == 0) {
            s_start = start;
            s_len = bad ? 0u : uint32_t(end - start);  // the offset chain bounds it by kTile
            s_bad = bad;
        }
    }
    __syncthreads();
    if (s_bad) {
        if (tid == 0) report(P.status, kStatusCorrupt);
        return;
    }

    // 3. stage the tile's exponent payload
    {
        const uint8_t* src = S + L.off_exp + s_start;
        const uint32_t len = s_len;
        for (uint32_t i = tid; i < len / 16; i += kThreads)
            *reinterpret_cast<uint4*>(s_exp + 16 * i) = ld_stream_v4(src + 16 * i);
        const uint32_t rem = len & 15u;
        if (tid < rem) s_exp[len - rem + tid] = src[len - rem + tid];
    }
    __syncthreads();

    // 4. decode 16 elements per chunk
    const uint32_t* s32 = reinterpret_cast<const uint32_t*>(s_exp);
#pragma unroll
    for (int k = 0; k < kChunksPerThread; ++k) {
        const uint32_t el = uint32_t(tid + k * kThreads) * kChunk;
        if (el >= tile_n) continue;
        const uint32_t blk = s_blk[el >> log2B];
        const uint32_t w = (blk >> 8) & 0xFFu;
        const OctetDecoder dec(w, blk & 0xFFu);
        const uint32_t q = (blk >> 16) + ((el & (B - 1)) >> 3) * w;
        uint32_t lo0, hi0, lo1, hi1;
        fetch_octet(s32, q, lo0, hi0);
        fetch_octet(s32, q + w, lo1, hi1);
        const uint4 r0 = dec.decode(lo0, hi0, M[k].x, M[k].y);
        const uint4 r1 = dec.decode(lo1, hi1, M[k].z, M[k].w);
        uint16_t* dst = I.out + tile_start + el;
        if (tile_n - el >= kChunk) {
            st_stream_v4(dst, r0);
            st_stream_v4(dst + 8, r1);
        } else {
            const uint32_t words[8] = {r0.x, r0.y, r0.z, r0.w, r1.x, r1.y, r1.z, r1.w};
            const uint32_t nv = tile_n - el;
            for (uint32_t i = 0; i < nv; ++i) dst[i] = uint16_t(words[i >> 1] >> (16 * (i & 1)));
        }
    }
}

template <int MAXI>
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
    if (tiles == 0) return cudaSuccess;
    decode_kernel<MAXI><<<unsigned(tiles), kThreads, 0, stream>>>(p);
    return cudaGetLastError();
}

}  // namespace

constexpr uint32_t kBatchMax = 512;

cudaError_t launch_decode(const DecodeItem* items, uint32_t count, int32_t* status,
                          cudaStream_t stream) {
    if (count == 1) return launch_batch<1>(items, 1, status, stream);
    for (uint32_t i = 0; i < count; i += kBatchMax) {
        const uint32_t c = min(kBatchMax, count - i);
        const cudaError_t err = launch_batch<kBatchMax>(items + i, c, status, stream);
        if (err != cudaSuccess) return err;
    }
    return cudaSuccess;
}

}  // namespace wc
