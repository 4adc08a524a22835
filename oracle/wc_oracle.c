/*
 * wc_oracle.c -- plain, slow, single-threaded CPU oracle for the WCB1 stream
 * (block fixed-length code of BF16 exponents, sign+mantissa bytes stored raw).
 *
 * TEST INFRASTRUCTURE. Only the test suite, the package smoke check and the
 * benchmark's CPU-baseline leg may load this file's library. The product path
 * (libwcodec) never calls it, and this file shares no code, header, table or
 * helper with the CUDA library: it is written separately from the stream
 * definition so that the two can be compared byte for byte.
 *
 * Source of the method: "ENEC: A Lossless AI Model Compression Method Enabling
 * Fast Inference on Ascend NPUs", Abstract. The abstract names the ingredients:
 * blocks coded at one fixed length each, a per-block bit width ("bit-width
 * quantization"), packing that combines values two, four, then eight at a time
 * ("hierarchical halving bit-packing"), a branch-free integer remap of the
 * values, and a prefix sum that places each block. It fixes no byte layout; the
 * layout below is this project's reading, and every such reading is marked.
 *
 * Encoding steps, in the order the abstract lists them:
 *   1. split each BF16 word into its exponent byte e = (x >> 7) & 0xFF and its
 *      sign+mantissa byte s = sign << 7 | mantissa   (reading: bit positions)
 *   2. bit-width quantization per block: lo = min e, hi = max e,
 *      w = bits(hi - lo) in 0..8; w == 8 is the raw fallback with base 0,
 *      otherwise base = lo                             (reading: remap = e - min)
 *   3. branch-free remap v = e - base
 *   4. hierarchical halving pack of each run of 8 values (an "octet") into
 *      w bytes, element t at bits [t*w, (t+1)*w), little-endian
 *   5. exclusive prefix sum of the block sizes ceil(L/8)*w -> block offsets
 *   6. write the sections: 128-byte container header, u16 block headers,
 *      u32 block offsets (16-byte units), mantissa plane, exponent plane;
 *      every section starts on a 128-byte boundary and all padding is zero.
 * Decoding is the exact inverse; its result is the input, bit for bit.
 *
 * FP32 tensors (reading: the same block scheme applied to the FP32 exponent):
 * the high half of an FP32 word has exactly the BF16 layout (sign, 8-bit
 * exponent, 7 mantissa bits), so the high halves are coded as above and the
 * low halves (16 more mantissa bits) are stored raw in a plane of their own
 * after the mantissa plane; the header's flags bit 0 marks such a stream.
 *
 * Escape-coded streams (reading; flags bit 1): a block's w-bit codes cover a
 * window of 2^w - 1 exponents [base, base + 2^w - 2] chosen for least size;
 * the code 2^w - 1 marks an element outside it, whose exponent byte goes to the
 * block's exception list right after its codes. "ZipServ: Fast and
 * Memory-Efficient LLM Inference with Hardware-Aware Lossless Compression",
 * Abstract, gives the direction (a fixed-length format with constant-time
 * parallel decoding that shrinks weights further); the window and escape
 * layout are this project's.
 */
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define ORC_OK 0
#define ORC_INVALID_ARG 1
#define ORC_BUFFER_TOO_SMALL 2
#define ORC_CORRUPT 3

#define ORC_MAGIC 0x31424357u /* the bytes "WCB1" read as a little-endian u32 */
#define ORC_FLAG_FP32 1u      /* header flags bit 0: an FP32 stream */
#define ORC_FLAG_ESCAPE 2u    /* header flags bit 1: an escape-coded stream */
#define ORC_VERSION 1u
#define ORC_HEADER_BYTES 128u
#define ORC_MAX_ELEMS (1ull << 36)

/* ------------------------------------------------------------------ */
/* Little-endian byte access (the stream is defined byte by byte).     */
/* ------------------------------------------------------------------ */
static void put_le(uint8_t *p, uint64_t value, int nbytes)
{
    for (int k = 0; k < nbytes; k++)
        p[k] = (uint8_t)(value >> (8 * k));
}

static uint64_t get_le(const uint8_t *p, int nbytes)
{
    uint64_t value = 0;
    for (int k = 0; k < nbytes; k++)
        value |= (uint64_t)p[k] << (8 * k);
    return value;
}

static uint64_t round_up_128(uint64_t x) { return (x + 127u) / 128u * 128u; }
static uint64_t round_up_16(uint64_t x) { return (x + 15u) / 16u * 16u; }

static int block_size_allowed(uint32_t B)
{
    /* reading: B is a power of two from 128 to 4096 */
    return B == 128 || B == 256 || B == 512 || B == 1024 || B == 2048 || B == 4096;
}

/* ------------------------------------------------------------------ */
/* Step 1: split and merge of one BF16 bit pattern.                    */
/* ------------------------------------------------------------------ */
uint8_t oracle_exponent(uint16_t x) { return (uint8_t)((x >> 7) & 0xFFu); }

uint8_t oracle_signman(uint16_t x)
{
    uint8_t sign = (uint8_t)(x >> 15);      /* bit 15 */
    uint8_t mantissa = (uint8_t)(x & 0x7Fu); /* bits 6..0 */
    return (uint8_t)((sign << 7) | mantissa);
}

uint16_t oracle_merge(uint8_t e, uint8_t s)
{
    uint16_t sign = (uint16_t)(s >> 7);
    uint16_t mantissa = (uint16_t)(s & 0x7Fu);
    return (uint16_t)((sign << 15) | ((uint16_t)e << 7) | mantissa);
}

/* ------------------------------------------------------------------ */
/* Step 2: bit-width quantization of one block.                        */
/* ------------------------------------------------------------------ */
/* The number of bits needed to write d in binary (0 for d == 0). */
unsigned oracle_bits(unsigned d)
{
    unsigned w = 0;
    while (d != 0) {
        w++;
        d >>= 1;
    }
    return w;
}

/* For the L words of one block: its width w and base. */
void oracle_block_params(const uint16_t *x, uint64_t L, uint8_t *base, uint8_t *w)
{
    unsigned lo = 255, hi = 0;
    for (uint64_t i = 0; i < L; i++) {
        unsigned e = oracle_exponent(x[i]);
        if (e < lo) lo = e;
        if (e > hi) hi = e;
    }
    if (L == 0) lo = hi = 0;
    unsigned width = oracle_bits(hi - lo);
    *w = (uint8_t)width;
    *base = (uint8_t)(width == 8 ? 0 : lo); /* raw fallback: the exponent itself */
}

/* ------------------------------------------------------------------ */
/* Step 4: hierarchical halving pack / unpack of one octet.            */
/* ------------------------------------------------------------------ */
static uint64_t low_mask(unsigned nbits)
{
    return nbits >= 64 ? ~0ull : ((1ull << nbits) - 1ull);
}

/* Pack 8 values of w bits: pairs, then quads, then the octet. */
uint64_t oracle_pack_octet(const uint8_t v[8], unsigned w)
{
    uint64_t pair[4], quad[2];
    for (int k = 0; k < 4; k++)
        pair[k] = (uint64_t)v[2 * k] | ((uint64_t)v[2 * k + 1] << w);
    for (int k = 0; k < 2; k++)
        quad[k] = pair[2 * k] | (pair[2 * k + 1] << (2 * w));
    return quad[0] | (quad[1] << (4 * w));
}

/* Undo the pack: the octet into quads, the quads into pairs, pairs into values. */
void oracle_unpack_octet(uint64_t octet, unsigned w, uint8_t v[8])
{
    uint64_t quad[2], pair[4];
    quad[0] = octet & low_mask(4 * w);
    quad[1] = (4 * w >= 64 ? 0 : octet >> (4 * w)) & low_mask(4 * w);
    for (int k = 0; k < 2; k++) {
        pair[2 * k] = quad[k] & low_mask(2 * w);
        pair[2 * k + 1] = (quad[k] >> (2 * w)) & low_mask(2 * w);
    }
    for (int k = 0; k < 4; k++) {
        v[2 * k] = (uint8_t)(pair[k] & low_mask(w));
        v[2 * k + 1] = (uint8_t)((pair[k] >> w) & low_mask(w));
    }
}

/* ------------------------------------------------------------------ */
/* Section layout, a function of (n, B) alone.                         */
/* ------------------------------------------------------------------ */
typedef struct {
    uint64_t nb, off_hdr, off_offs, off_man, off_low, off_exp;
} layout_t;

/* fp32 != 0: the stream of FP32 elements, whose high halves are coded as BF16
 * words and whose low halves follow the mantissa plane as a raw u16 plane
 * (reading: an FP32 word is a BF16 word followed by 16 more mantissa bits). */
static layout_t layout_of(uint64_t n, uint32_t B, int fp32)
{
    layout_t s;
    s.nb = (n + B - 1) / B;
    s.off_hdr = ORC_HEADER_BYTES;
    s.off_offs = s.off_hdr + round_up_128(2 * s.nb);
    s.off_man = s.off_offs + round_up_128(4 * s.nb);
    s.off_low = fp32 ? s.off_man + round_up_128(n) : 0;
    s.off_exp = fp32 ? s.off_low + round_up_128(2 * n) : s.off_man + round_up_128(n);
    return s;
}

static uint64_t block_len(uint64_t n, uint32_t B, uint64_t b)
{
    uint64_t start = b * (uint64_t)B;
    return (n - start < B) ? n - start : B;
}

/* Largest possible stream: every block raw (w = 8). 0 for a bad B or n. */
static uint64_t bound_impl(uint64_t n, uint32_t B, int fp32)
{
    if (!block_size_allowed(B) || n > ORC_MAX_ELEMS) return 0;
    layout_t s = layout_of(n, B, fp32);
    uint64_t worst = 0;
    for (uint64_t b = 0; b < s.nb; b++)
        worst += (block_len(n, B, b) + 7) / 8 * 8;
    return s.off_exp + worst;
}

uint64_t oracle_bound(uint64_t n, uint32_t B) { return bound_impl(n, B, 0); }
uint64_t oracle_bound_f32(uint64_t n, uint32_t B) { return bound_impl(n, B, 1); }

/* The 128-byte container header (the bytes after it are left as they are). */
static void write_container(uint8_t *out, uint32_t B, uint32_t flags, uint64_t n,
                            const layout_t *s, uint64_t E)
{
    memset(out, 0, ORC_HEADER_BYTES);
    put_le(out + 0, ORC_MAGIC, 4);
    put_le(out + 4, ORC_VERSION, 2);
    put_le(out + 6, ORC_HEADER_BYTES, 2);
    put_le(out + 8, B, 4);
    put_le(out + 12, flags, 4);
    put_le(out + 16, n, 8);
    put_le(out + 24, s->nb, 8);
    put_le(out + 32, s->off_hdr, 8);
    put_le(out + 40, s->off_offs, 8);
    put_le(out + 48, s->off_man, 8);
    put_le(out + 56, s->off_exp, 8);
    put_le(out + 64, E, 8);
    put_le(out + 72, s->off_exp + E, 8);
    put_le(out + 80, s->off_low, 8);
}

/* ------------------------------------------------------------------ */
/* Encoder.                                                            */
/* ------------------------------------------------------------------ */
/* x: the 16-bit words to code; lo: NULL, or the FP32 low halves (fp32 stream). */
static int compress_impl(const uint16_t *x, const uint16_t *lo, uint64_t n, uint32_t B,
                         uint8_t *out, uint64_t out_capacity, uint64_t *out_bytes)
{
    const int fp32 = lo != NULL;
    if (!block_size_allowed(B) || n > ORC_MAX_ELEMS || out == NULL ||
        out_bytes == NULL || (n > 0 && x == NULL))
        return ORC_INVALID_ARG;
    if (out_capacity < bound_impl(n, B, fp32)) return ORC_BUFFER_TOO_SMALL;

    layout_t s = layout_of(n, B, fp32);
    uint8_t *base = (uint8_t *)malloc(s.nb ? s.nb : 1);
    uint8_t *width = (uint8_t *)malloc(s.nb ? s.nb : 1);
    uint64_t *start = (uint64_t *)malloc((s.nb ? s.nb : 1) * sizeof(uint64_t));
    if (!base || !width || !start) {
        free(base);
        free(width);
        free(start);
        return ORC_INVALID_ARG;
    }

    /* Step 2: width and base of every block. */
    for (uint64_t b = 0; b < s.nb; b++)
        oracle_block_params(x + b * B, block_len(n, B, b), &base[b], &width[b]);

    /* Step 5: exclusive prefix sum of the block sizes, one block after another. */
    uint64_t running = 0;
    for (uint64_t b = 0; b < s.nb; b++) {
        start[b] = running;
        running += (block_len(n, B, b) + 7) / 8 * width[b];
    }
    uint64_t E = running;
    uint64_t total = s.off_exp + E;

    /* Step 6: sections; everything not written below stays zero. */
    memset(out, 0, total);
    write_container(out, B, fp32 ? ORC_FLAG_FP32 : 0u, n, &s, E);

    for (uint64_t b = 0; b < s.nb; b++) {
        put_le(out + s.off_hdr + 2 * b, (uint64_t)base[b] | ((uint64_t)width[b] << 8), 2);
        put_le(out + s.off_offs + 4 * b, start[b] / 16, 4);
    }

    /* Step 1 (mantissa half): the sign+mantissa bytes, in element order. */
    for (uint64_t i = 0; i < n; i++)
        out[s.off_man + i] = oracle_signman(x[i]);
    /* FP32: the low halves, raw, in element order. */
    if (fp32)
        for (uint64_t i = 0; i < n; i++) put_le(out + s.off_low + 2 * i, lo[i], 2);

    /* Steps 3 and 4: remap, then pack each octet into w bytes. */
    for (uint64_t b = 0; b < s.nb; b++) {
        uint64_t L = block_len(n, B, b);
        unsigned w = width[b];
        for (uint64_t j = 0; j < (L + 7) / 8; j++) {
            uint8_t v[8];
            for (int t = 0; t < 8; t++) {
                uint64_t k = 8 * j + (uint64_t)t;
                v[t] = (uint8_t)(k < L ? oracle_exponent(x[b * B + k]) - base[b] : 0);
            }
            put_le(out + s.off_exp + start[b] + j * w, oracle_pack_octet(v, w), (int)w);
        }
    }

    free(base);
    free(width);
    free(start);
    *out_bytes = total;
    return ORC_OK;
}

int oracle_compress(const uint16_t *x, uint64_t n, uint32_t B, uint8_t *out,
                    uint64_t out_capacity, uint64_t *out_bytes)
{
    return compress_impl(x, NULL, n, B, out, out_capacity, out_bytes);
}

/* FP32: split every word into its high half (a BF16 word: sign, 8-bit
 * exponent, 7 mantissa bits) and its low half (16 more mantissa bits). */
int oracle_compress_f32(const uint32_t *x, uint64_t n, uint32_t B, uint8_t *out,
                        uint64_t out_capacity, uint64_t *out_bytes)
{
    if (n > ORC_MAX_ELEMS || (n > 0 && x == NULL)) return ORC_INVALID_ARG;
    uint16_t *hi = (uint16_t *)malloc((n ? n : 1) * sizeof(uint16_t));
    uint16_t *lo = (uint16_t *)malloc((n ? n : 1) * sizeof(uint16_t));
    if (!hi || !lo) {
        free(hi);
        free(lo);
        return ORC_INVALID_ARG;
    }
    for (uint64_t i = 0; i < n; i++) {
        hi[i] = (uint16_t)(x[i] >> 16);
        lo[i] = (uint16_t)(x[i] & 0xFFFFu);
    }
    int rc = compress_impl(hi, lo, n, B, out, out_capacity, out_bytes);
    free(hi);
    free(lo);
    return rc;
}

/* ------------------------------------------------------------------ */
/* Decoder. Checks everything the stream definition fixes.             */
/* ------------------------------------------------------------------ */
static int all_zero(const uint8_t *p, uint64_t count)
{
    for (uint64_t k = 0; k < count; k++)
        if (p[k] != 0) return 0;
    return 1;
}

/* lo: NULL, or where the low halves of an FP32 stream go. */
static int decompress_impl(const uint8_t *in, uint64_t in_bytes, uint16_t *out, uint16_t *lo,
                           uint64_t n, uint32_t B)
{
    const int fp32 = lo != NULL;
    if (!block_size_allowed(B) || n > ORC_MAX_ELEMS || in == NULL || (n > 0 && out == NULL))
        return ORC_INVALID_ARG;
    if (in_bytes < ORC_HEADER_BYTES) return ORC_CORRUPT;

    layout_t s = layout_of(n, B, fp32);
    if (get_le(in + 0, 4) != ORC_MAGIC || get_le(in + 4, 2) != ORC_VERSION ||
        get_le(in + 6, 2) != ORC_HEADER_BYTES || get_le(in + 8, 4) != B ||
        get_le(in + 12, 4) != (uint64_t)fp32 || get_le(in + 16, 8) != n ||
        get_le(in + 24, 8) != s.nb || get_le(in + 32, 8) != s.off_hdr ||
        get_le(in + 40, 8) != s.off_offs || get_le(in + 48, 8) != s.off_man ||
        get_le(in + 56, 8) != s.off_exp || get_le(in + 80, 8) != s.off_low ||
        !all_zero(in + 88, 40))
        return ORC_CORRUPT;
    uint64_t E = get_le(in + 64, 8);
    uint64_t total = get_le(in + 72, 8);
    if (E > total || total != s.off_exp + E || total > in_bytes) return ORC_CORRUPT;

    /* Padding between sections must be zero. */
    if (!all_zero(in + s.off_hdr + 2 * s.nb, s.off_offs - s.off_hdr - 2 * s.nb) ||
        !all_zero(in + s.off_offs + 4 * s.nb, s.off_man - s.off_offs - 4 * s.nb))
        return ORC_CORRUPT;
    if (fp32 ? (!all_zero(in + s.off_man + n, s.off_low - s.off_man - n) ||
                !all_zero(in + s.off_low + 2 * n, s.off_exp - s.off_low - 2 * n))
             : !all_zero(in + s.off_man + n, s.off_exp - s.off_man - n))
        return ORC_CORRUPT;

    /* Headers and offsets must agree with the prefix sum of the block sizes. */
    uint64_t running = 0;
    for (uint64_t b = 0; b < s.nb; b++) {
        uint64_t h = get_le(in + s.off_hdr + 2 * b, 2);
        unsigned base = (unsigned)(h & 0xFFu), w = (unsigned)(h >> 8);
        if (w > 8 || (w == 8 && base != 0)) return ORC_CORRUPT;
        if (get_le(in + s.off_offs + 4 * b, 4) * 16 != running) return ORC_CORRUPT;
        running += (block_len(n, B, b) + 7) / 8 * w;
    }
    if (running != E) return ORC_CORRUPT;

    for (uint64_t b = 0; b < s.nb; b++) {
        uint64_t L = block_len(n, B, b);
        uint64_t h = get_le(in + s.off_hdr + 2 * b, 2);
        unsigned base = (unsigned)(h & 0xFFu), w = (unsigned)(h >> 8);
        uint64_t first = get_le(in + s.off_offs + 4 * b, 4) * 16;
        for (uint64_t j = 0; j < (L + 7) / 8; j++) {
            uint8_t v[8];
            oracle_unpack_octet(get_le(in + s.off_exp + first + j * w, (int)w), w, v);
            for (int t = 0; t < 8; t++) {
                uint64_t k = 8 * j + (uint64_t)t;
                if (k >= L) {
                    if (v[t] != 0) return ORC_CORRUPT; /* unused lanes are zero */
                    continue;
                }
                unsigned e = base + v[t];
                if (e > 255) return ORC_CORRUPT; /* no encoder writes such a value */
                out[b * B + k] = oracle_merge((uint8_t)e, in[s.off_man + b * B + k]);
            }
        }
    }
    if (fp32)
        for (uint64_t i = 0; i < n; i++) lo[i] = (uint16_t)get_le(in + s.off_low + 2 * i, 2);
    return ORC_OK;
}

int oracle_decompress(const uint8_t *in, uint64_t in_bytes, uint16_t *out,
                      uint64_t n, uint32_t B)
{
    return decompress_impl(in, in_bytes, out, NULL, n, B);
}

/* FP32: decode the high halves and the low plane, then join them. */
int oracle_decompress_f32(const uint8_t *in, uint64_t in_bytes, uint32_t *out,
                          uint64_t n, uint32_t B)
{
    if (n > ORC_MAX_ELEMS || (n > 0 && out == NULL)) return ORC_INVALID_ARG;
    uint16_t *hi = (uint16_t *)malloc((n ? n : 1) * sizeof(uint16_t));
    uint16_t *lo = (uint16_t *)malloc((n ? n : 1) * sizeof(uint16_t));
    if (!hi || !lo) {
        free(hi);
        free(lo);
        return ORC_INVALID_ARG;
    }
    int rc = decompress_impl(in, in_bytes, hi, lo, n, B);
    if (rc == ORC_OK)
        for (uint64_t i = 0; i < n; i++) out[i] = ((uint32_t)hi[i] << 16) | lo[i];
    free(hi);
    free(lo);
    return rc;
}

/* ------------------------------------------------------------------ */
/* Escape-coded streams (header flags bit 1).                          */
/* ------------------------------------------------------------------ */
/* Width w in 1..7: the window holds 2^w - 1 exponents and the code 2^w - 1
 * is the escape. base <= 255 - (2^w - 1), so base + code never exceeds 255. */
static unsigned escape_code(unsigned w) { return (1u << w) - 1u; }

static int in_window(unsigned e, unsigned base, unsigned w)
{
    return e >= base && e - base < escape_code(w);
}

/* (w, base) of one block of an escape-coded stream and its number of
 * exceptions K: the candidate of least cost ceil(L/8)*w + K among
 *   (0, e)        when every exponent of the block equals e,
 *   (w, base)     for 1 <= w <= 7 and 0 <= base <= 255 - (2^w - 1),
 *   (8, 0)        the raw block,
 * ties going to the smaller w, then to the larger base. */
void oracle_esc_block_params(const uint16_t *x, uint64_t L, uint8_t *base, uint8_t *w,
                             uint64_t *exceptions)
{
    uint64_t hist[256], below[257];
    memset(hist, 0, sizeof hist);
    for (uint64_t i = 0; i < L; i++) hist[oracle_exponent(x[i])]++;
    /* below[e] = number of elements with an exponent smaller than e */
    below[0] = 0;
    for (unsigned e = 0; e < 256; e++) below[e + 1] = below[e] + hist[e];

    const uint64_t octets = (L + 7) / 8;
    uint64_t best_cost = 8 * octets; /* the raw block, (8, 0) */
    unsigned best_w = 8, best_base = 0;
    uint64_t best_k = 0;
    for (unsigned e = 0; e < 256; e++)
        if (L > 0 && hist[e] == L) { /* one exponent only: (0, e) costs nothing */
            best_cost = 0, best_w = 0, best_base = e, best_k = 0;
        }
    for (unsigned ww = 1; ww <= 7; ww++) {
        const unsigned m = escape_code(ww);
        for (unsigned b = 0; b + m <= 255; b++) {
            const uint64_t inside = below[b + m] - below[b]; /* exponents b .. b + m - 1 */
            const uint64_t k = L - inside;
            const uint64_t cost = octets * ww + k;
            const int better = cost < best_cost ||
                               (cost == best_cost && ww < best_w) ||
                               (cost == best_cost && ww == best_w && b > best_base);
            if (better) best_cost = cost, best_w = ww, best_base = b, best_k = k;
        }
    }
    *w = (uint8_t)best_w;
    *base = (uint8_t)best_base;
    *exceptions = best_k;
}

/* Largest escape-coded stream: every block raw, each payload padded to 16 bytes. */
uint64_t oracle_bound_escape(uint64_t n, uint32_t B)
{
    if (!block_size_allowed(B) || n > ORC_MAX_ELEMS) return 0;
    layout_t s = layout_of(n, B, 0);
    uint64_t worst = 0;
    for (uint64_t b = 0; b < s.nb; b++) worst += round_up_16((block_len(n, B, b) + 7) / 8 * 8);
    return s.off_exp + worst;
}

int oracle_compress_escape(const uint16_t *x, uint64_t n, uint32_t B, uint8_t *out,
                           uint64_t out_capacity, uint64_t *out_bytes)
{
    if (!block_size_allowed(B) || n > ORC_MAX_ELEMS || out == NULL || out_bytes == NULL ||
        (n > 0 && x == NULL))
        return ORC_INVALID_ARG;
    if (out_capacity < oracle_bound_escape(n, B)) return ORC_BUFFER_TOO_SMALL;

    layout_t s = layout_of(n, B, 0);
    const uint64_t slots = s.nb ? s.nb : 1;
    uint8_t *base = (uint8_t *)malloc(slots);
    uint8_t *width = (uint8_t *)malloc(slots);
    uint64_t *start = (uint64_t *)malloc(slots * sizeof(uint64_t));
    uint64_t *nexc = (uint64_t *)malloc(slots * sizeof(uint64_t));
    if (!base || !width || !start || !nexc) {
        free(base);
        free(width);
        free(start);
        free(nexc);
        return ORC_INVALID_ARG;
    }

    /* Window, width and number of exceptions of every block. */
    for (uint64_t b = 0; b < s.nb; b++)
        oracle_esc_block_params(x + b * B, block_len(n, B, b), &base[b], &width[b], &nexc[b]);

    /* Exclusive prefix sum of the padded payload sizes. */
    uint64_t running = 0;
    for (uint64_t b = 0; b < s.nb; b++) {
        start[b] = running;
        running += round_up_16((block_len(n, B, b) + 7) / 8 * width[b] + nexc[b]);
    }
    const uint64_t E = running;
    const uint64_t total = s.off_exp + E;

    memset(out, 0, total);
    write_container(out, B, ORC_FLAG_ESCAPE, n, &s, E);
    for (uint64_t b = 0; b < s.nb; b++) {
        put_le(out + s.off_hdr + 2 * b, (uint64_t)base[b] | ((uint64_t)width[b] << 8), 2);
        put_le(out + s.off_offs + 4 * b, start[b] / 16, 4);
    }
    for (uint64_t i = 0; i < n; i++) out[s.off_man + i] = oracle_signman(x[i]);

    /* Codes, packed as in the plain stream, then the exception list. */
    for (uint64_t b = 0; b < s.nb; b++) {
        const uint64_t L = block_len(n, B, b);
        const unsigned w = width[b];
        uint8_t *payload = out + s.off_exp + start[b];
        uint8_t *exc = payload + (L + 7) / 8 * w;
        uint64_t k = 0;
        for (uint64_t j = 0; j < (L + 7) / 8; j++) {
            uint8_t c[8];
            for (int t = 0; t < 8; t++) {
                const uint64_t i = 8 * j + (uint64_t)t;
                c[t] = 0; /* lanes past the end of the block */
                if (i >= L) continue;
                const unsigned e = oracle_exponent(x[b * B + i]);
                if (w == 0) {
                    c[t] = 0; /* every exponent equals base: no code */
                } else if (w == 8) {
                    c[t] = (uint8_t)e; /* raw */
                } else if (in_window(e, base[b], w)) {
                    c[t] = (uint8_t)(e - base[b]);
                } else {
                    c[t] = (uint8_t)escape_code(w);
                    exc[k++] = (uint8_t)e;
                }
            }
            put_le(payload + j * w, oracle_pack_octet(c, w), (int)w);
        }
        (void)k; /* k == nexc[b] by construction of the block parameters */
    }

    free(base);
    free(width);
    free(start);
    free(nexc);
    *out_bytes = total;
    return ORC_OK;
}

int oracle_decompress_escape(const uint8_t *in, uint64_t in_bytes, uint16_t *out, uint64_t n,
                             uint32_t B)
{
    if (!block_size_allowed(B) || n > ORC_MAX_ELEMS || in == NULL || (n > 0 && out == NULL))
        return ORC_INVALID_ARG;
    if (in_bytes < ORC_HEADER_BYTES) return ORC_CORRUPT;

    layout_t s = layout_of(n, B, 0);
    if (get_le(in + 0, 4) != ORC_MAGIC || get_le(in + 4, 2) != ORC_VERSION ||
        get_le(in + 6, 2) != ORC_HEADER_BYTES || get_le(in + 8, 4) != B ||
        get_le(in + 12, 4) != ORC_FLAG_ESCAPE || get_le(in + 16, 8) != n ||
        get_le(in + 24, 8) != s.nb || get_le(in + 32, 8) != s.off_hdr ||
        get_le(in + 40, 8) != s.off_offs || get_le(in + 48, 8) != s.off_man ||
        get_le(in + 56, 8) != s.off_exp || get_le(in + 80, 8) != 0 || !all_zero(in + 88, 40))
        return ORC_CORRUPT;
    const uint64_t E = get_le(in + 64, 8);
    const uint64_t total = get_le(in + 72, 8);
    if (E > total || total != s.off_exp + E || total > in_bytes) return ORC_CORRUPT;
    if (!all_zero(in + s.off_hdr + 2 * s.nb, s.off_offs - s.off_hdr - 2 * s.nb) ||
        !all_zero(in + s.off_offs + 4 * s.nb, s.off_man - s.off_offs - 4 * s.nb) ||
        !all_zero(in + s.off_man + n, s.off_exp - s.off_man - n))
        return ORC_CORRUPT;

    const uint8_t *plane = in + s.off_exp;
    uint64_t running = 0; /* where the next block's payload must start */
    for (uint64_t b = 0; b < s.nb; b++) {
        const uint64_t L = block_len(n, B, b);
        const uint64_t h = get_le(in + s.off_hdr + 2 * b, 2);
        const unsigned base = (unsigned)(h & 0xFFu), w = (unsigned)(h >> 8);
        if (w > 8 || (w == 8 && base != 0)) return ORC_CORRUPT;
        if (w >= 1 && w <= 7 && base + escape_code(w) > 255) return ORC_CORRUPT;
        if (get_le(in + s.off_offs + 4 * b, 4) * 16 != running) return ORC_CORRUPT;
        const uint64_t code_bytes = (L + 7) / 8 * w;
        if (running + code_bytes > E) return ORC_CORRUPT;

        /* The codes; each escape takes the next exception byte. */
        const uint8_t *payload = plane + running;
        uint64_t k = 0;
        for (uint64_t j = 0; j < (L + 7) / 8; j++) {
            uint8_t c[8];
            oracle_unpack_octet(get_le(payload + j * w, (int)w), w, c);
            for (int t = 0; t < 8; t++) {
                const uint64_t i = 8 * j + (uint64_t)t;
                if (i >= L) {
                    if (c[t] != 0) return ORC_CORRUPT; /* unused lanes are zero */
                    continue;
                }
                unsigned e;
                if (w == 0) {
                    e = base;
                } else if (w == 8) {
                    e = c[t];
                } else if (c[t] != escape_code(w)) {
                    e = base + c[t];
                } else {
                    if (running + code_bytes + k >= E) return ORC_CORRUPT;
                    e = payload[code_bytes + k];
                    k++;
                    if (in_window(e, base, w)) return ORC_CORRUPT; /* not canonical */
                }
                out[b * B + i] = oracle_merge((uint8_t)e, in[s.off_man + b * B + i]);
            }
        }
        const uint64_t size = round_up_16(code_bytes + k);
        if (running + size > E) return ORC_CORRUPT;
        if (!all_zero(payload + code_bytes + k, size - code_bytes - k)) return ORC_CORRUPT;
        running += size;
    }
    if (running != E) return ORC_CORRUPT;
    return ORC_OK;
}

/* ------------------------------------------------------------------ */
/* tANS-coded streams (reading; flags bit 2).                          */
/* ------------------------------------------------------------------ */
/*
 * "MINE: Entropy-coded Memory-efficient Inference for Large Language Models",
 * Abstract: a GPU entropy coder of the tANS family (dtANS-LLM) that exploits
 * the non-uniform distribution of weight values and exposes hyper-parameters
 * trading compression ratio against decoding cost. The abstract gives no
 * format. Reading: the exponent bytes are coded by tabled asymmetric numeral
 * systems (Duda's tANS) over one normalized histogram per tensor, with L = 2^R
 * states; the sign+mantissa bytes stay raw as in every other stream kind.
 * The tensor is cut into chunks of C elements; a chunk is 32 interleaved lane
 * streams (lane l codes the chunk's elements l, l + 32, ...), each with its
 * own state, sharing one stream of 32-bit words that the lanes take in turn
 * (decode order: step by step, lanes in order). R and C are the
 * hyper-parameters.
 *
 * Layout: the WCB1 container header with flags = 4, the chunk size C in the
 * block-size field, nb = number of chunks and R in bytes 88..91;
 *   off_hdr  256 u16 normalized counts f[e] (sum L; all 0 when n = 0)
 *   off_offs nb u32 chunk offsets, 16-byte units, from off_exp
 *   off_man  n sign+mantissa bytes
 *   off_exp  per chunk: 32 u16 initial decoder states, then the u32 words,
 *            then zeros up to a multiple of 16 bytes
 * Decoding a lane: state X in [0, L); per element: refill when fewer than R
 * bits are buffered (the next word goes above the buffered bits), then
 * e = sym[X], X = next[X] + (the low nb[X] buffered bits), which are dropped.
 * A valid chunk ends with every state 0 and has fewer than 4 unused words.
 */
#define ORC_FLAG_TANS 4u
#define ORC_TANS_LANES 32u

static int tans_chunk_allowed(uint32_t C)
{
    return C == 1024 || C == 2048 || C == 4096 || C == 8192; /* reading */
}

static int tans_log_allowed(uint32_t R) { return R >= 8 && R <= 12; } /* reading */

static unsigned floor_log2(uint32_t v)
{
    unsigned k = 0;
    while ((v >> (k + 1)) != 0) k++;
    return k;
}

/* Normalize exponent counts to a sum of L = 2^R (reading of the
 * normalization, which the page leaves open): every present exponent gets
 * max(1, floor(count * L / total)); the shortfall goes to, and any excess
 * comes off, the entry with the largest normalized count (the smaller
 * exponent on ties), one at a time. */
void oracle_tans_normalize(const uint64_t counts[256], uint32_t R, uint16_t freq[256])
{
    const uint32_t L = 1u << R;
    uint64_t total = 0;
    for (int e = 0; e < 256; e++) total += counts[e];
    uint64_t sum = 0;
    for (int e = 0; e < 256; e++) {
        uint64_t f = 0;
        if (counts[e] > 0) {
            f = counts[e] * L / total;
            if (f == 0) f = 1;
        }
        freq[e] = (uint16_t)f;
        sum += f;
    }
    if (total == 0) return;
    while (sum != L) {
        int big = 0;
        for (int e = 1; e < 256; e++)
            if (freq[e] > freq[big]) big = e;
        if (sum < L) {
            freq[big]++;
            sum++;
        } else {
            freq[big]--;
            sum--;
        }
    }
}

/* Decoding table of the normalized counts (sum L): the exponents are spread
 * over the L states with the odd step L/2 + L/8 + 3 (which visits every
 * state once), then state X holding the v-th occurrence of e (v counted from
 * f[e]) decodes to e with nb = R - floor(log2 v) bits and next = v * 2^nb - L.
 * pos[e][v - f[e]] = X is the encoder's inverse map (pos_base[e] indexes it). */
static void tans_tables(const uint16_t freq[256], uint32_t R, uint8_t *sym, uint8_t *nbits,
                        uint16_t *next, uint16_t *pos, uint32_t pos_base[256])
{
    const uint32_t L = 1u << R, step = (L >> 1) + (L >> 3) + 3;
    uint32_t p = 0, acc = 0;
    for (int e = 0; e < 256; e++) {
        pos_base[e] = acc;
        acc += freq[e];
        for (uint32_t i = 0; i < freq[e]; i++) {
            sym[p] = (uint8_t)e;
            p = (p + step) & (L - 1);
        }
    }
    uint32_t seen[256];
    for (int e = 0; e < 256; e++) seen[e] = freq[e];
    for (uint32_t X = 0; X < L; X++) {
        const unsigned e = sym[X];
        const uint32_t v = seen[e]++;
        const unsigned nb = R - floor_log2(v);
        nbits[X] = (uint8_t)nb;
        next[X] = (uint16_t)((v << nb) - L);
        pos[pos_base[e] + (v - freq[e])] = (uint16_t)X;
    }
}

/* The decoding table alone (for the tests): sym, nb and next of every state. */
void oracle_tans_table(const uint16_t freq[256], uint32_t R, uint8_t *sym, uint8_t *nbits,
                       uint16_t *next)
{
    uint16_t *pos = malloc(2 * ((size_t)1 << R));
    uint32_t pos_base[256];
    if (pos == NULL) return;
    tans_tables(freq, R, sym, nbits, next, pos, pos_base);
    free(pos);
}

static uint64_t tans_chunk_len(uint64_t n, uint32_t C, uint64_t c)
{
    const uint64_t start = c * (uint64_t)C;
    return (n - start < C) ? n - start : C;
}

typedef struct {
    uint64_t nb, off_hdr, off_offs, off_man, off_exp;
} tans_layout_t;

static tans_layout_t tans_layout(uint64_t n, uint32_t C)
{
    tans_layout_t s;
    s.nb = (n + C - 1) / C;
    s.off_hdr = ORC_HEADER_BYTES;
    s.off_offs = s.off_hdr + 512;
    s.off_man = s.off_offs + round_up_128(4 * s.nb);
    s.off_exp = s.off_man + round_up_128(n);
    return s;
}

/* Words of one lane: the refill rule can buffer at most R - 1 bits before a
 * refill and consumes at most R bits per element, so a lane of k elements
 * takes at most 1 + floor(k * R / (33 - R)) words (each refill is followed by
 * at least 33 - R consumed bits before the next). */
uint64_t oracle_bound_tans(uint64_t n, uint32_t C, uint32_t R)
{
    if (!tans_chunk_allowed(C) || !tans_log_allowed(R) || n > ORC_MAX_ELEMS) return 0;
    tans_layout_t s = tans_layout(n, C);
    uint64_t worst = 0;
    for (uint64_t c = 0; c < s.nb; c++) {
        const uint64_t len = tans_chunk_len(n, C, c);
        const uint64_t k = (len + ORC_TANS_LANES - 1) / ORC_TANS_LANES;
        const uint64_t words = ORC_TANS_LANES * (1 + k * R / (33 - R));
        worst += round_up_16(2 * ORC_TANS_LANES + 4 * words);
    }
    return s.off_exp + worst;
}

int oracle_compress_tans(const uint16_t *x, uint64_t n, uint32_t C, uint32_t R, uint8_t *out,
                         uint64_t out_capacity, uint64_t *out_bytes)
{
    if (!tans_chunk_allowed(C) || !tans_log_allowed(R) || n > ORC_MAX_ELEMS || out == NULL ||
        out_bytes == NULL || (n > 0 && x == NULL))
        return ORC_INVALID_ARG;
    if (out_capacity < oracle_bound_tans(n, C, R)) return ORC_BUFFER_TOO_SMALL;
    const uint32_t L = 1u << R;
    tans_layout_t s = tans_layout(n, C);
    memset(out, 0, s.off_exp);

    /* the histogram of the exponents and its normalization */
    uint64_t counts[256] = {0};
    for (uint64_t i = 0; i < n; i++) counts[oracle_exponent(x[i])]++;
    uint16_t freq[256];
    oracle_tans_normalize(counts, R, freq);
    for (int e = 0; e < 256; e++) put_le(out + s.off_hdr + 2 * e, freq[e], 2);
    for (uint64_t i = 0; i < n; i++) out[s.off_man + i] = oracle_signman(x[i]);

    uint8_t *sym = malloc(L), *nbits = malloc(L);
    uint16_t *next = malloc(2 * (size_t)L), *pos = malloc(2 * (size_t)L);
    uint16_t *val = malloc(2 * (size_t)C);
    uint8_t *len_bits = malloc(C);
    /* a lane's words: at most 1 + floor(k * R / (33 - R)) for k elements */
    const uint64_t lane_cap = 2 + (uint64_t)(C / ORC_TANS_LANES) * R / (33 - R);
    uint32_t *lane_words = malloc(4 * (size_t)lane_cap * ORC_TANS_LANES);
    uint32_t pos_base[256];
    if (!sym || !nbits || !next || !pos || !val || !len_bits || !lane_words) {
        free(sym); free(nbits); free(next); free(pos); free(val); free(len_bits);
        free(lane_words);
        return ORC_INVALID_ARG;
    }
    tans_tables(freq, R, sym, nbits, next, pos, pos_base);

    uint64_t running = 0;
    for (uint64_t c = 0; c < s.nb; c++) {
        const uint64_t first = c * (uint64_t)C, len = tans_chunk_len(n, C, c);
        uint8_t *payload = out + s.off_exp + running;
        put_le(out + s.off_offs + 4 * c, running / 16, 4);
        /* 1. every lane coded backwards from its last element: each element
         *    gives the bits its decoding will read (value, count), element by
         *    element in chunk order */
        for (uint32_t l = 0; l < ORC_TANS_LANES; l++) {
            uint32_t state = L; /* the encoder's state lives in [L, 2L) */
            const uint64_t steps = len > l ? (len - l + ORC_TANS_LANES - 1) / ORC_TANS_LANES : 0;
            for (uint64_t k = steps; k-- > 0;) {
                const uint64_t i = l + k * ORC_TANS_LANES;
                const unsigned e = oracle_exponent(x[first + i]);
                const uint32_t f = freq[e];
                unsigned nb = 0;
                while ((state >> nb) >= 2 * f) nb++;
                val[i] = (uint16_t)(state & ((1u << nb) - 1u));
                len_bits[i] = (uint8_t)nb;
                state = L + pos[pos_base[e] + ((state >> nb) - f)];
            }
            put_le(payload + 2 * l, state - L, 2); /* the decoder's first state */
        }
        /* 2. each lane's bits in element order, bit by bit, 32 to a word */
        uint64_t lane_bits[ORC_TANS_LANES] = {0};
        for (uint32_t l = 0; l < ORC_TANS_LANES; l++) {
            uint32_t *lw = lane_words + (uint64_t)l * lane_cap;
            memset(lw, 0, 4 * (size_t)lane_cap);
            for (uint64_t j = l; j < len; j += ORC_TANS_LANES)
                for (unsigned b = 0; b < len_bits[j]; b++, lane_bits[l]++)
                    if ((val[j] >> b) & 1u) lw[lane_bits[l] / 32] |= 1u << (lane_bits[l] % 32);
        }
        /* 3. the words, in the order the decoder takes them: step by step,
         *    lanes in order, a lane refilling when it holds fewer than R bits */
        uint64_t words = 0;
        uint32_t cnt[ORC_TANS_LANES] = {0};   /* bits buffered by the decoder */
        uint64_t taken[ORC_TANS_LANES] = {0}; /* words of the lane already taken */
        const uint64_t max_steps = (len + ORC_TANS_LANES - 1) / ORC_TANS_LANES;
        for (uint64_t k = 0; k < max_steps; k++) {
            for (uint32_t l = 0; l < ORC_TANS_LANES; l++) {
                const uint64_t i = l + k * ORC_TANS_LANES;
                if (i >= len || cnt[l] >= R) continue;
                if (2 * ORC_TANS_LANES + 4 * (words + 1) > out_capacity - s.off_exp - running ||
                    taken[l] >= lane_cap) {
                    free(sym); free(nbits); free(next); free(pos); free(val); free(len_bits);
                    free(lane_words);
                    return ORC_BUFFER_TOO_SMALL;
                }
                put_le(payload + 2 * ORC_TANS_LANES + 4 * words,
                       lane_words[(uint64_t)l * lane_cap + taken[l]], 4);
                words++;
                taken[l]++;
                cnt[l] += 32;
            }
            for (uint32_t l = 0; l < ORC_TANS_LANES; l++) {
                const uint64_t i = l + k * ORC_TANS_LANES;
                if (i < len) cnt[l] -= len_bits[i];
            }
        }
        const uint64_t size = round_up_16(2 * ORC_TANS_LANES + 4 * words);
        memset(payload + 2 * ORC_TANS_LANES + 4 * words, 0,
               size - 2 * ORC_TANS_LANES - 4 * words);
        running += size;
    }
    free(sym); free(nbits); free(next); free(pos); free(val); free(len_bits);
    free(lane_words);

    layout_t hdr;
    hdr.nb = s.nb;
    hdr.off_hdr = s.off_hdr;
    hdr.off_offs = s.off_offs;
    hdr.off_man = s.off_man;
    hdr.off_low = 0;
    hdr.off_exp = s.off_exp;
    write_container(out, C, ORC_FLAG_TANS, n, &hdr, running);
    put_le(out + 88, R, 4);
    *out_bytes = s.off_exp + running;
    return ORC_OK;
}

int oracle_decompress_tans(const uint8_t *in, uint64_t in_bytes, uint16_t *out, uint64_t n,
                           uint32_t C)
{
    if (!tans_chunk_allowed(C) || n > ORC_MAX_ELEMS || in == NULL || (n > 0 && out == NULL))
        return ORC_INVALID_ARG;
    if (in_bytes < ORC_HEADER_BYTES) return ORC_CORRUPT;
    tans_layout_t s = tans_layout(n, C);
    const uint32_t R = (uint32_t)get_le(in + 88, 4);
    if (get_le(in + 0, 4) != ORC_MAGIC || get_le(in + 4, 2) != ORC_VERSION ||
        get_le(in + 6, 2) != ORC_HEADER_BYTES || get_le(in + 8, 4) != C ||
        get_le(in + 12, 4) != ORC_FLAG_TANS || get_le(in + 16, 8) != n ||
        get_le(in + 24, 8) != s.nb || get_le(in + 32, 8) != s.off_hdr ||
        get_le(in + 40, 8) != s.off_offs || get_le(in + 48, 8) != s.off_man ||
        get_le(in + 56, 8) != s.off_exp || get_le(in + 80, 8) != 0 ||
        !tans_log_allowed(R) || !all_zero(in + 92, 36))
        return ORC_CORRUPT;
    const uint64_t E = get_le(in + 64, 8);
    const uint64_t total = get_le(in + 72, 8);
    if (E > total || total != s.off_exp + E || total > in_bytes) return ORC_CORRUPT;
    if (!all_zero(in + s.off_offs + 4 * s.nb, s.off_man - s.off_offs - 4 * s.nb) ||
        !all_zero(in + s.off_man + n, s.off_exp - s.off_man - n))
        return ORC_CORRUPT;
    const uint32_t L = 1u << R;
    uint16_t freq[256];
    uint64_t sum = 0;
    for (int e = 0; e < 256; e++) {
        freq[e] = (uint16_t)get_le(in + s.off_hdr + 2 * e, 2);
        sum += freq[e];
    }
    if (sum != (n > 0 ? L : 0)) return ORC_CORRUPT;
    if (n == 0) return E == 0 ? ORC_OK : ORC_CORRUPT;

    uint8_t *sym = malloc(L), *nbits = malloc(L);
    uint16_t *next = malloc(2 * (size_t)L), *pos = malloc(2 * (size_t)L);
    uint32_t pos_base[256];
    if (!sym || !nbits || !next || !pos) {
        free(sym); free(nbits); free(next); free(pos);
        return ORC_INVALID_ARG;
    }
    tans_tables(freq, R, sym, nbits, next, pos, pos_base);
    int rc = ORC_OK;
    uint64_t running = 0;
    for (uint64_t c = 0; c < s.nb && rc == ORC_OK; c++) {
        const uint64_t first = c * (uint64_t)C, len = tans_chunk_len(n, C, c);
        const uint64_t start = 16 * get_le(in + s.off_offs + 4 * c, 4);
        const uint64_t end = c + 1 < s.nb ? 16 * get_le(in + s.off_offs + 4 * (c + 1), 4) : E;
        if (start != running || end < start + 2 * ORC_TANS_LANES || end > E) {
            rc = ORC_CORRUPT;
            break;
        }
        const uint8_t *payload = in + s.off_exp + start;
        const uint64_t avail = (end - start - 2 * ORC_TANS_LANES) / 4;
        uint32_t X[ORC_TANS_LANES], cnt[ORC_TANS_LANES];
        uint64_t buf[ORC_TANS_LANES];
        for (uint32_t l = 0; l < ORC_TANS_LANES; l++) {
            X[l] = (uint32_t)get_le(payload + 2 * l, 2);
            cnt[l] = 0;
            buf[l] = 0;
            if (X[l] >= L || (l >= len && X[l] != 0)) rc = ORC_CORRUPT;
        }
        uint64_t words = 0;
        const uint64_t max_steps = (len + ORC_TANS_LANES - 1) / ORC_TANS_LANES;
        for (uint64_t k = 0; k < max_steps && rc == ORC_OK; k++) {
            for (uint32_t l = 0; l < ORC_TANS_LANES; l++) {
                const uint64_t i = l + k * ORC_TANS_LANES;
                if (i >= len) continue;
                if (cnt[l] < R) {
                    if (words >= avail) {
                        rc = ORC_CORRUPT;
                        break;
                    }
                    buf[l] |= get_le(payload + 2 * ORC_TANS_LANES + 4 * words, 4) << cnt[l];
                    cnt[l] += 32;
                    words++;
                }
            }
            for (uint32_t l = 0; l < ORC_TANS_LANES && rc == ORC_OK; l++) {
                const uint64_t i = l + k * ORC_TANS_LANES;
                if (i >= len) continue;
                const unsigned nb = nbits[X[l]];
                const unsigned e = sym[X[l]];
                X[l] = next[X[l]] + (uint32_t)(buf[l] & ((1u << nb) - 1u));
                buf[l] >>= nb;
                cnt[l] -= nb;
                out[first + i] = oracle_merge((uint8_t)e, in[s.off_man + first + i]);
            }
        }
        if (rc != ORC_OK) break;
        /* every lane back at state 0, no bits left over, padding zero */
        for (uint32_t l = 0; l < ORC_TANS_LANES; l++)
            if (X[l] != 0 || buf[l] != 0) rc = ORC_CORRUPT;
        if (avail - words > 3 ||
            !all_zero(payload + 2 * ORC_TANS_LANES + 4 * words,
                      end - start - 2 * ORC_TANS_LANES - 4 * words))
            rc = ORC_CORRUPT;
        running = end;
    }
    if (rc == ORC_OK && running != E) rc = ORC_CORRUPT;
    free(sym); free(nbits); free(next); free(pos);
    return rc;
}
