// wc_escape_core.cuh -- decoding steps of escape-coded WCB1 streams (sm_100a).
//
// An escape-coded block (header flags bit 1) codes the exponents of a window of
// 2^w - 1 values [base, base + 2^w - 2] at w bits each; the code 2^w - 1 is an
// escape, and the exponent bytes of the escaped elements follow the block's
// codes, in element order, as its exception list. The codes are packed by
// hierarchical halving exactly like a plain block ("ENEC: A Lossless AI Model
// Compression Method Enabling Fast Inference on Ascend NPUs", Abstract), so an
// element's code still sits at a closed-form position; only an escaped
// element's exception needs a count of the escapes before it in its block.
// The direction -- a fixed-length format that decodes in constant time, in
// parallel, and shrinks weights further -- is that of "ZipServ: Fast and
// Memory-Efficient LLM Inference with Hardware-Aware Lossless Compression",
// Abstract; the window and escape layout are this library's.
//
// base <= 255 - (2^w - 1) for 1 <= w <= 7, so base + code fits a byte for
// every code, escape included: a word of four codes takes its base with one
// 32-bit add.
#pragma once

#include "wc_decode_core.cuh"

namespace wc {

// Bytes [q, q + 2W) of the staged codes of one 16-element chunk, as a little-
// endian bit string in X[0..3]. q is 2W * (chunk index in its block) past a
// 16-byte boundary: 4-byte aligned for even W, 2-byte aligned for odd W.
template <int W>
__device__ __forceinline__ void fetch_chunk_bits(const uint8_t* exp, uint32_t q, uint32_t X[4]) {
    if constexpr (W == 1) {
        X[0] = *reinterpret_cast<const uint16_t*>(exp + q);
    } else if constexpr (W == 2) {
        X[0] = *reinterpret_cast<const uint32_t*>(exp + q);
    } else if constexpr (W == 4) {
        const uint2 v = *reinterpret_cast<const uint2*>(exp + q);
        X[0] = v.x;
        X[1] = v.y;
    } else if constexpr (W == 6) {
        const uint32_t* s32 = reinterpret_cast<const uint32_t*>(exp + q);
        X[0] = s32[0];
        X[1] = s32[1];
        X[2] = s32[2];
    } else {  // odd W >= 3: 2W bytes from a 2-byte boundary
        const uint32_t* s32 = reinterpret_cast<const uint32_t*>(exp + (q & ~3u));
        const uint32_t r = (q & 2u) * 8u;  // 0 or 16
        constexpr int kWords = (2 * W + 2 + 3) / 4;  // words that cover [q, q + 2W)
        uint32_t x[kWords + 1];
#pragma unroll
        for (int k = 0; k < kWords; ++k) x[k] = s32[k];
        x[kWords] = 0;
#pragma unroll
        for (int k = 0; k < kWords; ++k) X[k] = __funnelshift_r(x[k], x[k + 1], r);
    }
}

// Quad j of a chunk: bits [4Wj, 4Wj + 4W) of X (4W <= 28 bits).
template <int W, int J>
__device__ __forceinline__ uint32_t chunk_quad(const uint32_t X[4]) {
    constexpr int kPos = 4 * W * J, kWord = kPos / 32, kOff = kPos % 32;
    uint32_t v;
    if constexpr (kOff == 0)
        v = X[kWord];
    else if constexpr (kOff + 4 * W <= 32)
        v = X[kWord] >> kOff;
    else
        v = __funnelshift_r(X[kWord], X[kWord + 1], kOff);
    return v & ((1u << (4 * W)) - 1u);
}

// Reverse the halving of one quad: quad -> two pairs in 16-bit lanes -> four
// values in bytes (value t of the quad in byte t).
template <int W>
__device__ __forceinline__ uint32_t quad_to_bytes(uint32_t Q) {
    constexpr uint32_t M2 = (1u << (2 * W)) - 1u, m1 = (1u << W) - 1u;
    if constexpr (W <= 4) {  // the shifted copies cannot reach the kept bits
        const uint32_t t = (Q | (Q << (16 - 2 * W))) & (M2 | (M2 << 16));
        return (t | (t << (8 - W))) & (m1 * 0x01010101u);
    } else {
        const uint32_t t = (Q & M2) | ((Q << (16 - 2 * W)) & (M2 << 16));
        return (t & (m1 * 0x00010001u)) | ((t << (8 - W)) & (m1 * 0x01000100u));
    }
}

// The 16 codes of a chunk as exponent bytes: E[j] holds elements 4j..4j+3
// (base added; escaped elements hold base + 2^W - 1 until patched), and
// esc[j] has bit 8t+7 set when element 4j+t is escaped.
template <int W>
__device__ __forceinline__ void chunk_exponents(const uint8_t* exp, uint32_t q, uint32_t base4,
                                                uint32_t esc_add, uint32_t E[4], uint32_t esc[4]) {
    if constexpr (W == 0) {
#pragma unroll
        for (int j = 0; j < 4; ++j) E[j] = base4, esc[j] = 0u;
    } else if constexpr (W == 8) {  // raw block: the codes are the exponents
        const uint4 v = *reinterpret_cast<const uint4*>(exp + q);
        E[0] = v.x;
        E[1] = v.y;
        E[2] = v.z;
        E[3] = v.w;
#pragma unroll
        for (int j = 0; j < 4; ++j) esc[j] = 0u;
    } else {
        uint32_t X[4] = {0u, 0u, 0u, 0u};
        fetch_chunk_bits<W>(exp, q, X);
        uint32_t V[4];
        V[0] = quad_to_bytes<W>(chunk_quad<W, 0>(X));
        V[1] = quad_to_bytes<W>(chunk_quad<W, 1>(X));
        V[2] = quad_to_bytes<W>(chunk_quad<W, 2>(X));
        V[3] = quad_to_bytes<W>(chunk_quad<W, 3>(X));
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            // a byte equals 2^W - 1 (the largest value it can hold) exactly when
            // adding 0x80 - (2^W - 1) sets its top bit; no carries leave a byte
            esc[j] = (V[j] + esc_add) & 0x80808080u;
            E[j] = V[j] + base4;
        }
    }
}

// chunk_exponents for a width known only at run time (0..8), the same result:
// the chunk's two octets are fetched as 64-bit strings, each split into two
// quads, each quad spread into bytes with run-time shifts.
__device__ __forceinline__ void chunk_exponents_rt(const uint8_t* exp, uint32_t q, uint32_t w,
                                                   uint32_t base4, uint32_t esc_add, uint32_t E[4],
                                                   uint32_t esc[4]) {
    if (w == 0u) {
#pragma unroll
        for (int j = 0; j < 4; ++j) E[j] = base4, esc[j] = 0u;
        return;
    }
    const uint32_t* s32 = reinterpret_cast<const uint32_t*>(exp);
    uint32_t lo[2], hi[2];
    fetch_octet(s32, q, lo[0], hi[0]);
    fetch_octet(s32, q + w, lo[1], hi[1]);
    const uint32_t w4 = 4u * w;
    const uint32_t m4 = w == 8u ? 0xFFFFFFFFu : (1u << w4) - 1u;
    const uint32_t M2 = (1u << (2u * w)) - 1u, m1x2 = ((1u << w) - 1u) * 0x00010001u;
    const uint32_t sh2 = 16u - 2u * w, sh1 = 8u - w;
    // raw blocks (w = 8) hold any byte: they have no escape code
    const uint32_t detect = w == 8u ? 0u : 0x80808080u;
#pragma unroll
    for (int k = 0; k < 2; ++k) {
        const uint32_t Q[2] = {lo[k] & m4, __funnelshift_rc(lo[k], hi[k], w4) & m4};
#pragma unroll
        for (int h = 0; h < 2; ++h) {
            const uint32_t t = (Q[h] & M2) | ((Q[h] << sh2) & (M2 << 16));
            const uint32_t V = (t & m1x2) | ((t << sh1) & (m1x2 << 8));
            esc[2 * k + h] = (V + esc_add) & detect;
            E[2 * k + h] = V + base4;
        }
    }
}

// The escapes of a chunk: their number, from the four escape words at once
// (their flag bits are moved to distinct positions and counted together).
__device__ __forceinline__ uint32_t escape_count(const uint32_t esc[4]) {
    return __popc(esc[0] | (esc[1] >> 1) | (esc[2] >> 2) | (esc[3] >> 3));
}

// ... and their mask, bit t for element t: bits 7, 15, 23, 31 of a word go to
// bits 28..31 of one product (its other bits do not overlap, so nothing
// carries into them), then into place.
__device__ __forceinline__ uint32_t escape_mask(const uint32_t esc[4]) {
    uint32_t m16 = 0;
#pragma unroll
    for (int j = 0; j < 4; ++j) m16 |= ((esc[j] * 0x00204081u) >> 28) << (4 * j);
    return m16;
}

__device__ __forceinline__ void chunk_exponents_w(uint32_t w, const uint8_t* exp, uint32_t q,
                                                  uint32_t base4, uint32_t esc_add, uint32_t E[4],
                                                  uint32_t esc[4]) {
    switch (w) {
        case 0: chunk_exponents<0>(exp, q, base4, esc_add, E, esc); break;
        case 1: chunk_exponents<1>(exp, q, base4, esc_add, E, esc); break;
        case 2: chunk_exponents<2>(exp, q, base4, esc_add, E, esc); break;
        case 3: chunk_exponents<3>(exp, q, base4, esc_add, E, esc); break;
        case 4: chunk_exponents<4>(exp, q, base4, esc_add, E, esc); break;
        case 5: chunk_exponents<5>(exp, q, base4, esc_add, E, esc); break;
        case 6: chunk_exponents<6>(exp, q, base4, esc_add, E, esc); break;
        case 7: chunk_exponents<7>(exp, q, base4, esc_add, E, esc); break;
        default: chunk_exponents<8>(exp, q, base4, esc_add, E, esc); break;
    }
}

// Four exponent bytes (elements 4j..4j+3) and their four sign+mantissa bytes
// -> two words of two BF16 each: x = (s & 0x80) << 8 | e << 7 | (s & 0x7F).
__device__ __forceinline__ void merge_quad(uint32_t E, uint32_t S, uint32_t& lo, uint32_t& hi) {
    lo = prmt(E, 0u, 0x4140u) * 128u + (prmt(S, 0u, 0x1100u) & 0x807F807Fu);
    hi = prmt(E, 0u, 0x4342u) * 128u + (prmt(S, 0u, 0x3322u) & 0x807F807Fu);
}

// Check a tile's block metadata for an escape-coded stream and write each
// block's decode constants:
//   t0 = {payload start within the staged bytes, w, code bytes ceil(L/8)*w,
//         payload end within the staged bytes}
//   t1 = {base * 0x01010101, (0x80 - (2^w - 1)) * 0x01010101 for 1 <= w <= 7}
// Checks: w <= 8; base 0 when w == 8; base + 2^w - 1 <= 255 when 1 <= w <= 7;
// every payload holds its codes and is no longer than a raw block's (16-byte
// padded); the tile's payload inside stream_bytes. The exact payload size
// (which depends on the number of escapes) is checked by the decoding warps.
// [start, start + len16) is left for a bulk copy, as in commit_tile_meta.
// Called by all 32 lanes of a warp.
__device__ inline bool commit_tile_meta_escape(const TileMeta& m, const uint8_t* S,
                                               const Layout& L, uint64_t stream_bytes,
                                               uint32_t tile_n, uint4* t0, uint2* t1,
                                               uint8_t* exp_stage, uint64_t& start,
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
            const uint64_t octets = (len + 7) >> 3;
            bad |= w > 8u || (w == 8u && base != 0u);
            bad |= w >= 1u && w <= 7u && base + (1u << w) - 1u > 255u;
            // an unsigned difference: a payload that ends before it starts fails too
            bad |= m.nx[j] < m.sb[j] + octets * min(w, 8u);
            bad |= m.nx[j] - m.sb[j] > ((8 * octets + 15) & ~uint64_t(15));
        }
    }
    bad |= end > stream_bytes - L.off_exp;
    bad = __any_sync(0xFFFFFFFFu, bad);
    if (bad) return false;
    // every payload is at most its raw size, so end - start <= kTile + 8
#pragma unroll
    for (int j = 0; j < 2; ++j) {
        const uint32_t b = lane + 32 * j;
        if (b < nblk) {
            const uint32_t w = m.h[j] >> 8, base = m.h[j] & 0xFFu;
            const uint32_t len = min(B, tile_n - b * B);
            const uint32_t m1 = (1u << w) - 1u;
            t0[b] = make_uint4(uint32_t(m.sb[j] - start), w, ((len + 7) >> 3) * w,
                               uint32_t(m.nx[j] - start));
            t1[b] = make_uint2(base * 0x01010101u,
                               (w >= 1u && w <= 7u) ? (0x80u - m1) * 0x01010101u : 0u);
        }
    }
    const uint32_t len = uint32_t(end - start);
    len16 = len & ~15u;
    const uint32_t rem = len - len16;  // 0 for a well-formed stream
    if (uint32_t(lane) < rem) exp_stage[len16 + lane] = S[L.off_exp + start + len16 + lane];
    return true;
}

}  // namespace wc
