// wc_pack_core.cuh -- the per-element split and the hierarchical halving pack
// shared by the encoders (sm_100a): "ENEC: A Lossless AI Model Compression
// Method Enabling Fast Inference on Ascend NPUs", Abstract (byte-level split,
// branch-free remap, values packed two, four, then eight at a time).
#pragma once

#include "wc_internal.cuh"

namespace wc {

// Four BF16 words (two u32) -> their four sign+mantissa bytes and their four
// exponent bytes, in element order. lo/hi gather the words' low and high
// bytes; s = hi's bit 7 (the sign) over lo's bits 6..0 (the mantissa);
// e = hi's bits 6..0 above lo's bit 7 (the exponent, bits 14..7 of the word).
__device__ __forceinline__ void split_quad(uint32_t x01, uint32_t x23, uint32_t& s4,
                                           uint32_t& e4) {
    const uint32_t lo = prmt(x01, x23, 0x6420u), hi = prmt(x01, x23, 0x7531u);
    s4 = (hi & 0x80808080u) | (lo & 0x7F7F7F7Fu);
    e4 = ((hi << 1) & 0xFEFEFEFEu) | ((lo >> 7) & 0x01010101u);
}

// Hierarchical halving with a compile-time width W: four W-bit values (the
// bytes of v) -> two pairs of 2W bits -> one quad of 4W bits.
template <uint32_t W>
__device__ __forceinline__ uint32_t pack_quad(uint32_t v) {
    const uint32_t pairs = (v & 0x00FF00FFu) | (((v >> 8) & 0x00FF00FFu) << W);
    return (pairs & 0xFFFFu) | ((pairs >> 16) << (2 * W));
}

// A 16-element chunk at width W: four quads -> two octets -> the chunk's 2W
// bytes (element t at bits [t*W, t*W + W)), stored little-endian at dst. dst
// is a multiple of 2W bytes past a 16-byte boundary, so the widest aligned
// store follows from W: one 16-byte store at W = 8, 8 bytes at W = 4, 4 at
// W = 2, three 4-byte stores at W = 6, 2-byte stores for odd W.
template <uint32_t W>
__device__ __forceinline__ void pack_chunk(const uint32_t V[4], uint8_t* dst) {
    if constexpr (W == 0) {
        return;
    } else if constexpr (W == 4) {
        // values below 16: v | v >> 4 holds pair 0 (v0 | v1 << 4) in byte 0 and
        // pair 1 in byte 2 (the shifted copies land only in bytes 1 and 3), and
        // the four pairs of two words are their octet's bytes in order
        uint32_t p[4];
#pragma unroll
        for (uint32_t j = 0; j < 4; ++j) p[j] = V[j] | (V[j] >> 4);
        *reinterpret_cast<uint2*>(dst) = make_uint2(prmt(p[0], p[1], 0x6420u), prmt(p[2], p[3], 0x6420u));
    } else {
        uint32_t F[4] = {0u, 0u, 0u, 0u};
#pragma unroll
        for (uint32_t j = 0; j < 4; ++j) {
            const uint32_t q = pack_quad<W>(V[j]);
            constexpr uint32_t kBits = 4 * W;
            const uint32_t pos = j * kBits, word = pos / 32, off = pos % 32;
            F[word] |= q << off;
            if (off != 0 && off + kBits > 32) F[word + 1] |= q >> (32 - off);
        }
        if constexpr (W == 8) {
            *reinterpret_cast<uint4*>(dst) = make_uint4(F[0], F[1], F[2], F[3]);
        } else if constexpr (W == 4) {
            *reinterpret_cast<uint2*>(dst) = make_uint2(F[0], F[1]);
        } else if constexpr (W == 2) {
            *reinterpret_cast<uint32_t*>(dst) = F[0];
        } else if constexpr (W == 6) {
            uint32_t* d = reinterpret_cast<uint32_t*>(dst);
            d[0] = F[0];
            d[1] = F[1];
            d[2] = F[2];
        } else {
            uint16_t* d = reinterpret_cast<uint16_t*>(dst);
#pragma unroll
            for (uint32_t m = 0; m < W; ++m) d[m] = uint16_t(F[m / 2] >> (16 * (m % 2)));
        }
    }
}

__device__ __forceinline__ void pack_chunk_w(uint32_t w, const uint32_t V[4], uint8_t* dst) {
    switch (w) {
        case 1: pack_chunk<1>(V, dst); break;
        case 2: pack_chunk<2>(V, dst); break;
        case 3: pack_chunk<3>(V, dst); break;
        case 4: pack_chunk<4>(V, dst); break;
        case 5: pack_chunk<5>(V, dst); break;
        case 6: pack_chunk<6>(V, dst); break;
        case 7: pack_chunk<7>(V, dst); break;
        case 8: pack_chunk<8>(V, dst); break;
        default: break;  // w = 0: no exponent bytes
    }
}

// The ragged end of a tensor: the chunk's first nbytes bytes only, one at a
// time (lanes past the end already hold 0).
__device__ inline void pack_chunk_tail(uint32_t w, const uint32_t V[4], uint8_t* dst, uint32_t nbytes) {
    for (uint32_t i = 0; i < nbytes; ++i) {
        uint32_t byte = 0;
        for (uint32_t bit = 0; bit < 8; ++bit) {  // bit 8i+bit of the chunk's field
            const uint32_t pos = 8 * i + bit, t = pos / w, within = pos % w;
            const uint32_t v = (V[t / 4] >> (8 * (t % 4))) & 0xFFu;
            byte |= ((v >> within) & 1u) << bit;
        }
        dst[i] = uint8_t(byte);
    }
}

}  // namespace wc
