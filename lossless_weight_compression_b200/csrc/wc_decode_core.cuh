// wc_decode_core.cuh -- the per-octet decoding steps shared by the decoder and
// the fused decode-GEMV kernels (sm_100a). Element t of an octet sits at bits
// [t*w, (t+1)*w) of the octet's w bytes ("ENEC: A Lossless AI Model Compression
// Method Enabling Fast Inference on Ascend NPUs", Abstract: hierarchical
// halving packing; reversed here octet -> quads -> pairs -> values).
#pragma once

#include "wc_internal.cuh"

namespace wc {

// 64 bits starting at byte q of the staged exponent bytes (q need not be aligned).
__device__ __forceinline__ void fetch_octet(const uint32_t* s32, uint32_t q, uint32_t& lo,
                                            uint32_t& hi) {
    const uint32_t a = q >> 2, r = (q & 3u) * 8u;
    const uint32_t x0 = s32[a], x1 = s32[a + 1], x2 = s32[a + 2];
    lo = __funnelshift_r(x0, x1, r);
    hi = __funnelshift_r(x1, x2, r);
}

// A pair (2w bits, v0 | v1 << w) -> both 16-bit lanes' exponent fields (base + v) << 7.
__device__ __forceinline__ uint32_t pair_lanes(uint32_t p, uint32_t sh, uint32_t M1,
                                               uint32_t base7) {
    return ((p | (p << sh)) & M1) * 128u + base7;
}

// Octet (lo:hi, bits above 8w ignored) + 8 sign+mantissa bytes -> 8 BF16 words.
//   quads: bits [0,4w) and [4w,8w); pairs: the halves of each quad.
// A sign+mantissa byte replicated into both bytes of a lane and masked with
// 0x807F leaves the mantissa in bits 0..6 and the sign in bit 15.
__device__ __forceinline__ uint4 decode_octet(uint32_t lo, uint32_t hi, uint32_t s03,
                                              uint32_t s47, uint32_t w2, uint32_t w4,
                                              uint32_t sh, uint4 t1) {
    const uint32_t M1 = t1.x, m2 = t1.y, m4 = t1.z, base7 = t1.w;
    const uint32_t p0 = lo & m2;
    const uint32_t p1 = __funnelshift_r(lo, hi, w2) & m2;
    const uint32_t q1 = __funnelshift_rc(lo, hi, w4) & m4;
    const uint32_t p2 = q1 & m2;
    const uint32_t p3 = q1 >> w2;
    uint4 r;
    r.x = (prmt(s03, 0u, 0x1100u) & 0x807F807Fu) | pair_lanes(p0, sh, M1, base7);
    r.y = (prmt(s03, 0u, 0x3322u) & 0x807F807Fu) | pair_lanes(p1, sh, M1, base7);
    r.z = (prmt(s47, 0u, 0x1100u) & 0x807F807Fu) | pair_lanes(p2, sh, M1, base7);
    r.w = (prmt(s47, 0u, 0x3322u) & 0x807F807Fu) | pair_lanes(p3, sh, M1, base7);
    return r;
}

// The common case w = 4: an octet is 4 bytes, element t in nibble t. Low
// nibbles give the even elements, high nibbles the odd ones; a byte permute
// then places elements 2k and 2k+1 in the two 16-bit lanes of a word, using
// the permute's sign-replicating selectors on bytes below 0x80 as zero bytes.
// Same result as decode_octet. Two octets f0, f1 with their sign+mantissa
// bytes in M.xy and M.zw:
__device__ __forceinline__ void decode_octets_w4(uint32_t f0, uint32_t f1, uint4 M, uint32_t base7,
                                                 uint4& r0, uint4& r1) {
    const uint32_t e0 = f0 & 0x0F0F0F0Fu, o0 = (f0 >> 4) & 0x0F0F0F0Fu;  // octet 0
    const uint32_t e1 = f1 & 0x0F0F0F0Fu, o1 = (f1 >> 4) & 0x0F0F0F0Fu;  // octet 1
    r0.x = (prmt(M.x, 0u, 0x1100u) & 0x807F807Fu) | (prmt(e0, o0, 0xC480u) * 128u + base7);
    r0.y = (prmt(M.x, 0u, 0x3322u) & 0x807F807Fu) | (prmt(e0, o0, 0xD591u) * 128u + base7);
    r0.z = (prmt(M.y, 0u, 0x1100u) & 0x807F807Fu) | (prmt(e0, o0, 0xE6A2u) * 128u + base7);
    r0.w = (prmt(M.y, 0u, 0x3322u) & 0x807F807Fu) | (prmt(e0, o0, 0xF7B3u) * 128u + base7);
    r1.x = (prmt(M.z, 0u, 0x1100u) & 0x807F807Fu) | (prmt(e1, o1, 0xC480u) * 128u + base7);
    r1.y = (prmt(M.z, 0u, 0x3322u) & 0x807F807Fu) | (prmt(e1, o1, 0xD591u) * 128u + base7);
    r1.z = (prmt(M.w, 0u, 0x1100u) & 0x807F807Fu) | (prmt(e1, o1, 0xE6A2u) * 128u + base7);
    r1.w = (prmt(M.w, 0u, 0x3322u) & 0x807F807Fu) | (prmt(e1, o1, 0xF7B3u) * 128u + base7);
}

// One chunk of 16 elements at w = 4: its two octets are the 8 bytes at q
// (8-byte aligned: q = payload offset + 4 * (element offset in the block / 8)).
__device__ __forceinline__ void decode_chunk_w4(const uint8_t* exp_stage, uint32_t q, uint4 M,
                                                uint32_t base7, uint4& r0, uint4& r1) {
    const uint2 F = *reinterpret_cast<const uint2*>(exp_stage + q);
    decode_octets_w4(F.x, F.y, M, base7, r0, r1);
}

// Two octets of any width (0..8) starting at bytes q0 and q1 of the staged
// exponent bytes, with their sign+mantissa bytes in M.xy and M.zw.
__device__ __forceinline__ void decode_octets_any(const uint8_t* exp_stage, uint32_t q0, uint32_t q1,
                                                  uint4 M, uint4 t0, uint4 t1, uint4& r0, uint4& r1) {
    const uint32_t* s32 = reinterpret_cast<const uint32_t*>(exp_stage);
    const uint32_t sh = 16u - t0.y;
    uint32_t lo0, hi0, lo1, hi1;
    fetch_octet(s32, q0, lo0, hi0);
    fetch_octet(s32, q1, lo1, hi1);
    r0 = decode_octet(lo0, hi0, M.x, M.y, t0.z, t0.w, sh, t1);
    r1 = decode_octet(lo1, hi1, M.z, M.w, t0.z, t0.w, sh, t1);
}

// One chunk of 16 elements at any width (0..8), as two octets through decode_octet.
__device__ __forceinline__ void decode_chunk_any(const uint8_t* exp_stage, uint32_t q, uint4 M,
                                                 uint4 t0, uint4 t1, uint4& r0, uint4& r1) {
    decode_octets_any(exp_stage, q, q + t0.y, M, t0, t1, r0, r1);
}

// One chunk of 16 elements at any width: the w = 4 path above, else two octets
// through decode_octet.
__device__ __forceinline__ void decode_chunk(const uint8_t* exp_stage, uint32_t q, uint4 M,
                                            uint4 t0, uint4 t1, uint4& r0, uint4& r1) {
    if (t0.y == 4u)
        decode_chunk_w4(exp_stage, q, M, t1.w, r0, r1);
    else
        decode_chunk_any(exp_stage, q, M, t0, t1, r0, r1);
}

__device__ __forceinline__ uint64_t ld_u64(const uint8_t* p) {
    return *reinterpret_cast<const uint64_t*>(p);
}

// The first tile of each tensor checks the container header against (n, B).
__device__ inline void check_container(const DecodeItem& I, const Layout& L, int32_t* status) {
    const uint8_t* S = I.stream;
    bool bad = ld_u64(S) != (kMagic | (uint64_t(kVersion) << 32) | (uint64_t(kHeaderBytes) << 48));
    bad |= ld_u64(S + 8) != (uint64_t(L.block) | (uint64_t(L.flags) << 32));  // block size, flags
    bad |= ld_u64(S + 16) != L.n;
    bad |= ld_u64(S + 24) != L.nb;
    bad |= ld_u64(S + 32) != L.off_hdr;
    bad |= ld_u64(S + 40) != L.off_offs;
    bad |= ld_u64(S + 48) != L.off_man;
    bad |= ld_u64(S + 56) != L.off_exp;
    const uint64_t E = ld_u64(S + 64), total = ld_u64(S + 72);
    bad |= E > L.n + 16 || total != L.off_exp + E || total > I.stream_bytes;
    bad |= ld_u64(S + 80) != L.off_low;
    for (int k = 88; k < 128; k += 8) bad |= ld_u64(S + k) != 0;
    if (bad) report(status, kStatusCorrupt);
}

// Block metadata of one tile (the tile covering elements [first, first + tile_n)
// of a stream: whole blocks, at most 64), as each lane of a warp holds it:
// lane l owns blocks l and l + 32 (header, payload start, next block's start).
struct TileMeta {
    uint32_t h[2];
    uint64_t sb[2], nx[2];
};

// Issue the loads of a tile's block headers and offsets. The values are only
// used by commit_tile_meta, so a producer can load the next tile's metadata
// while it waits for a free stage for the current one.
__device__ __forceinline__ TileMeta load_tile_meta(const uint8_t* S, const Layout& L,
                                                   uint64_t first, uint32_t tile_n, int lane) {
    TileMeta m;
    const uint32_t log2B = L.log2_block, B = L.block;
    const uint64_t b0 = first >> log2B;
    const uint32_t nblk = (tile_n + B - 1) >> log2B;
    const uint16_t* hdr = reinterpret_cast<const uint16_t*>(S + L.off_hdr) + b0;
    const uint32_t* offs = reinterpret_cast<const uint32_t*>(S + L.off_offs) + b0;
#pragma unroll
    for (int j = 0; j < 2; ++j) {
        const uint32_t b = lane + 32 * j;
        m.h[j] = 0;
        m.sb[j] = m.nx[j] = 0;
        if (b < nblk) {
            m.h[j] = hdr[b];
            m.sb[j] = 16ull * offs[b];
            m.nx[j] = (b + 1 < nblk || b0 + b + 1 < L.nb) ? 16ull * offs[b + 1]
                                                          : ld_u64(S + 64);  // E
        }
    }
    return m;
}

// Check a tile's metadata: every w <= 8, base 0 when w == 8, offsets equal to
// the prefix sum of the block sizes, and the payload inside stream_bytes.
// Writes each block's decode constants into t0/t1 (t0 = {payload offset within
// the tile, w, 2w, 4w}, t1 = {m1 | m1 << 16, m2, m4, base * 0x00800080},
// mk = 2^k - 1) and the payload's bytes past its last 16-byte boundary (only at
// the very end of a stream) into exp_stage. Returns false if the metadata
// breaks the stream definition; otherwise [start, start + len16) is the
// 16-byte-aligned part of the tile's exponent payload, left for a bulk copy.
// Called by all 32 lanes of a warp.
__device__ inline bool commit_tile_meta(const TileMeta& m, const uint8_t* S, const Layout& L,
                                        uint64_t stream_bytes, uint32_t tile_n, uint4* t0,
                                        uint4* t1, uint8_t* exp_stage, uint64_t& start,
                                        uint32_t& len16, int lane) {
    const uint32_t log2B = L.log2_block, B = L.block;
    const uint32_t nblk = (tile_n + B - 1) >> log2B;
    start = __shfl_sync(0xFFFFFFFFu, m.sb[0], 0);
    const uint32_t last = nblk - 1;
    const uint64_t end = __shfl_sync(0xFFFFFFFFu, last < 32 ? m.nx[0] : m.nx[1], last & 31);
    bool bad = false;
#pragma unroll
    for (int j = 0; j < 2; ++j) {
        const uint32_t b = lane + 32 * j;
        if (b < nblk) {
            const uint32_t w = m.h[j] >> 8, base = m.h[j] & 0xFFu;
            const uint32_t len = min(B, tile_n - b * B);
            bad |= w > 8u || (w == 8u && base != 0u);
            bad |= m.sb[j] + uint64_t((len + 7) >> 3) * min(w, 8u) != m.nx[j];
        }
    }
    bad |= end > stream_bytes - L.off_exp;
    bad = __any_sync(0xFFFFFFFFu, bad);
    if (bad) return false;
    // the offset chain holds, so end - start = the tile's payload <= kTile
#pragma unroll
    for (int j = 0; j < 2; ++j) {
        const uint32_t b = lane + 32 * j;
        if (b < nblk) {
            const uint32_t w = m.h[j] >> 8, base = m.h[j] & 0xFFu;
            const uint32_t m1 = (1u << w) - 1u;
            t0[b] = make_uint4(uint32_t(m.sb[j] - start), w, 2 * w, 4 * w);
            t1[b] = make_uint4(m1 | (m1 << 16), (1u << (2 * w)) - 1u,
                               w == 8u ? 0xFFFFFFFFu : (1u << (4 * w)) - 1u, base * 0x00800080u);
        }
    }
    const uint32_t len = uint32_t(end - start);
    len16 = len & ~15u;
    const uint32_t rem = len - len16;  // only at the very end of a stream
    if (uint32_t(lane) < rem) exp_stage[len16 + lane] = S[L.off_exp + start + len16 + lane];
    return true;
}

}  // namespace wc
