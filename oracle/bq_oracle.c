/*
 * bq_oracle.c - plain CPU reference (see bq_oracle.h for what it follows).
 *
 * TEST INFRASTRUCTURE ONLY: used by tests/, the package smoke check and the
 * benchmark's CPU-baseline leg; never by the library path.
 *
 * Build: gcc -std=c11 -O2 -ffp-contract=off -fno-fast-math -fPIC -shared
 * (see oracle/build.py).  The code is a direct transcription of the method's
 * definitions, one element at a time, with no blocking, vectorisation or
 * reordering of the arithmetic.
 */
#include "bq_oracle.h"

#include <math.h>
#include <string.h>

/* ---------------------------------------------------------------- types -- */

static float bits_to_f32(uint32_t u) { float f; memcpy(&f, &u, 4); return f; }
static uint32_t f32_to_bits(float f) { uint32_t u; memcpy(&u, &f, 4); return u; }

/* IEEE binary16 -> binary32, exact (every binary16 value is a binary32 value). */
float bqo_f16_to_f32(uint16_t h)
{
    int sign = h >> 15;
    int e = (h >> 10) & 31;
    int m = h & 1023;
    float v;
    if (e == 0)
        v = ldexpf((float)m, -24);                 /* zero or subnormal: m * 2^-24 */
    else if (e == 31)
        v = m ? NAN : INFINITY;
    else
        v = ldexpf((float)(m + 1024), e - 25);     /* (1024 + m) * 2^(e - 15 - 10) */
    return sign ? -v : v;
}

/* bfloat16 is the top half of a binary32. */
float bqo_bf16_to_f32(uint16_t h) { return bits_to_f32((uint32_t)h << 16); }

/* binary32 -> bfloat16, round to nearest, ties to even. */
uint16_t bqo_f32_to_bf16(float f)
{
    uint32_t u = f32_to_bits(f);
    if ((u & 0x7fffffffu) > 0x7f800000u)           /* NaN: keep it a quiet NaN */
        return (uint16_t)((u >> 16) | 0x40u);
    uint32_t lower = u & 0xffffu;
    uint32_t upper = u >> 16;
    if (lower > 0x8000u || (lower == 0x8000u && (upper & 1u)))
        upper += 1;                                /* carries into the exponent */
    return (uint16_t)upper;
}

/* binary32 -> binary16, round to nearest, ties to even. */
uint16_t bqo_f32_to_f16(float f)
{
    uint32_t u = f32_to_bits(f);
    uint16_t sign = (uint16_t)((u >> 16) & 0x8000u);
    uint32_t a = u & 0x7fffffffu;
    if (a > 0x7f800000u)
        return (uint16_t)(sign | 0x7e00u);         /* NaN */
    if (a >= 0x477ff000u)                          /* >= 65520: rounds to infinity */
        return (uint16_t)(sign | 0x7c00u);
    if (a < 0x38800000u) {                         /* below 2^-14: subnormal range */
        /* the result is round(|f| * 2^24) units of 2^-24; the product is exact
         * in double and nearbyint rounds ties to even */
        double units = nearbyint((double)fabsf(f) * 16777216.0);
        return (uint16_t)(sign | (uint16_t)units); /* 1024 is the smallest normal */
    }
    /* normal: rebias the exponent (127 -> 15) and drop 13 mantissa bits */
    uint32_t h = (a - 0x38000000u) >> 13;
    uint32_t rem = a & 0x1fffu;
    if (rem > 0x1000u || (rem == 0x1000u && (h & 1u)))
        h += 1;
    return (uint16_t)(sign | h);
}

static float load_elem(const void *x, int dtype, int64_t i)
{
    switch (dtype) {
    case BQO_F32:  return ((const float *)x)[i];
    case BQO_F16:  return bqo_f16_to_f32(((const uint16_t *)x)[i]);
    default:       return bqo_bf16_to_f32(((const uint16_t *)x)[i]);
    }
}

static void store_elem(void *y, int dtype, int64_t i, float v)
{
    switch (dtype) {
    case BQO_F32:  ((float *)y)[i] = v; break;
    case BQO_F16:  ((uint16_t *)y)[i] = bqo_f32_to_f16(v); break;
    default:       ((uint16_t *)y)[i] = bqo_f32_to_bf16(v); break;
    }
}

static int valid_dtype(int d) { return d == BQO_F32 || d == BQO_F16 || d == BQO_BF16; }

static int valid_blocksize(int bs)
{
    /* bitsandbytes PR #2052: every block size from 32 through 4096 */
    return bs >= 32 && bs <= 4096 && (bs & (bs - 1)) == 0;
}

/* ------------------------------------------------------ nearest code ---- */

/*
 * Nearest-code search as the plain definition: the distance to entry j is
 * |RN(xn - code[j])| in binary32; the smallest distance wins and, on equal
 * distances, the lowest index wins (strict "<" while scanning upwards).
 */
int bqo_nearest_code(float xn, const float *code, int entries)
{
    int idx = 0;
    float best = fabsf(xn - code[0]);
    for (int j = 1; j < entries; ++j) {
        float d = fabsf(xn - code[j]);
        if (d < best) {
            best = d;
            idx = j;
        }
    }
    return idx;
}

/* ---------------------------------------------------------- quantize ---- */

int bqo_quantize_blockwise(const void *x, int dtype, int64_t n, int blocksize,
                           const float *code, int entries,
                           float *absmax, uint8_t *out)
{
    if (n < 0 || !valid_dtype(dtype) || !valid_blocksize(blocksize) ||
        (entries != 16 && entries != 256))
        return -1;
    if (n == 0)
        return 0;
    int64_t nb = (n + blocksize - 1) / blocksize;
    int64_t out_bytes = entries == 16 ? (n + 1) / 2 : n;
    memset(out, 0, (size_t)out_bytes);

    for (int64_t b = 0; b < nb; ++b) {
        int64_t lo = b * blocksize;
        int64_t hi = lo + blocksize < n ? lo + blocksize : n;

        /* step 1: absmax over the block's valid elements */
        float A = 0.0f;
        for (int64_t i = lo; i < hi; ++i)
            A = fmaxf(A, fabsf(load_elem(x, dtype, i)));
        absmax[b] = A;

        /* step 2: normalise by IEEE division, search the codebook, pack */
        for (int64_t i = lo; i < hi; ++i) {
            float v = load_elem(x, dtype, i);
            float xn = (A == 0.0f) ? 0.0f : v / A;
            int idx = bqo_nearest_code(xn, code, entries);
            if (entries == 16) {
                if ((i & 1) == 0)
                    out[i >> 1] |= (uint8_t)(idx << 4);   /* element 2i: high nibble */
                else
                    out[i >> 1] |= (uint8_t)idx;          /* element 2i+1: low nibble */
            } else {
                out[i] = (uint8_t)idx;
            }
        }
    }
    return 0;
}

/* -------------------------------------------------------- dequantize ---- */

int bqo_dequantize_blockwise(const uint8_t *q, const float *absmax, int64_t n,
                             int blocksize, const float *code, int entries,
                             void *y, int ydtype)
{
    if (n < 0 || !valid_dtype(ydtype) || !valid_blocksize(blocksize) ||
        (entries != 16 && entries != 256))
        return -1;
    for (int64_t i = 0; i < n; ++i) {
        int idx;
        if (entries == 16)
            idx = (i & 1) ? (q[i >> 1] & 15) : (q[i >> 1] >> 4);
        else
            idx = q[i];
        float v = code[idx] * absmax[i / blocksize];
        store_elem(y, ydtype, i, v);
    }
    return 0;
}

/* -------------------------------------------------------------- GGUF ---- */

static float block_scale(const uint8_t *blk)
{
    return bqo_f16_to_f32((uint16_t)(blk[0] | (blk[1] << 8)));
}

int bqo_dequant_q8_0(const uint8_t *blocks, int64_t n_blocks, void *y, int ydtype)
{
    if (n_blocks < 0 || !valid_dtype(ydtype))
        return -1;
    for (int64_t k = 0; k < n_blocks; ++k) {
        const uint8_t *blk = blocks + 34 * k;
        float d = block_scale(blk);
        for (int j = 0; j < 32; ++j) {
            int qv = (int)(int8_t)blk[2 + j];
            store_elem(y, ydtype, 32 * k + j, d * (float)qv);
        }
    }
    return 0;
}

int bqo_dequant_q4_0(const uint8_t *blocks, int64_t n_blocks, void *y, int ydtype)
{
    if (n_blocks < 0 || !valid_dtype(ydtype))
        return -1;
    for (int64_t k = 0; k < n_blocks; ++k) {
        const uint8_t *blk = blocks + 18 * k;
        float d = block_scale(blk);
        for (int j = 0; j < 16; ++j) {
            int lo = blk[2 + j] & 15;      /* shift 0: elements 0..15  */
            int hi = blk[2 + j] >> 4;      /* shift 4: elements 16..31 */
            store_elem(y, ydtype, 32 * k + j, d * (float)(lo - 8));
            store_elem(y, ydtype, 32 * k + 16 + j, d * (float)(hi - 8));
        }
    }
    return 0;
}

/* ------------------------------------------------------- more GGUF types -- */

static float half_at(const uint8_t *p) { return bqo_f16_to_f32((uint16_t)(p[0] | (p[1] << 8))); }

static uint32_t u32_at(const uint8_t *p)
{
    return (uint32_t)p[0] | ((uint32_t)p[1] << 8) | ((uint32_t)p[2] << 16) | ((uint32_t)p[3] << 24);
}

int bqo_dequant_q4_1(const uint8_t *blocks, int64_t n_blocks, void *y, int ydtype)
{
    if (n_blocks < 0 || !valid_dtype(ydtype))
        return -1;
    for (int64_t k = 0; k < n_blocks; ++k) {
        const uint8_t *blk = blocks + 20 * k;
        float d = half_at(blk), m = half_at(blk + 2);
        for (int j = 0; j < 16; ++j) {
            int lo = blk[4 + j] & 15, hi = blk[4 + j] >> 4;
            store_elem(y, ydtype, 32 * k + j, d * (float)lo + m);
            store_elem(y, ydtype, 32 * k + 16 + j, d * (float)hi + m);
        }
    }
    return 0;
}

/* 5-bit value of element e (0..31) of a Q5 block: nibble plus bit e of qh */
static int q5_value(const uint8_t *qs, uint32_t qh, int e)
{
    int nib = e < 16 ? (qs[e] & 15) : (qs[e - 16] >> 4);
    return nib | (int)(((qh >> e) & 1u) << 4);
}

int bqo_dequant_q5_0(const uint8_t *blocks, int64_t n_blocks, void *y, int ydtype)
{
    if (n_blocks < 0 || !valid_dtype(ydtype))
        return -1;
    for (int64_t k = 0; k < n_blocks; ++k) {
        const uint8_t *blk = blocks + 22 * k;
        float d = half_at(blk);
        uint32_t qh = u32_at(blk + 2);
        for (int e = 0; e < 32; ++e)
            store_elem(y, ydtype, 32 * k + e, d * (float)(q5_value(blk + 6, qh, e) - 16));
    }
    return 0;
}

int bqo_dequant_q5_1(const uint8_t *blocks, int64_t n_blocks, void *y, int ydtype)
{
    if (n_blocks < 0 || !valid_dtype(ydtype))
        return -1;
    for (int64_t k = 0; k < n_blocks; ++k) {
        const uint8_t *blk = blocks + 24 * k;
        float d = half_at(blk), m = half_at(blk + 2);
        uint32_t qh = u32_at(blk + 4);
        for (int e = 0; e < 32; ++e)
            store_elem(y, ydtype, 32 * k + e, d * (float)q5_value(blk + 8, qh, e) + m);
    }
    return 0;
}

/* Q4_K: the 6-bit scale and min of sub-block i from the 12 packed bytes:
 * sub-blocks 0..3 keep theirs in the low 6 bits of bytes i and i + 4;
 * sub-blocks 4..7 take their low 4 bits from byte i + 4 (scale: low nibble,
 * min: high nibble) and their top 2 bits from the top 2 bits of bytes i - 4
 * (scale) and i (min). */
static void q4k_scale_min(const uint8_t *sc, int i, int *scale, int *mn)
{
    if (i < 4) {
        *scale = sc[i] & 63;
        *mn = sc[i + 4] & 63;
    } else {
        *scale = (sc[i + 4] & 15) | ((sc[i - 4] >> 6) << 4);
        *mn = (sc[i + 4] >> 4) | ((sc[i] >> 6) << 4);
    }
}

int bqo_dequant_q4_k(const uint8_t *blocks, int64_t n_blocks, void *y, int ydtype)
{
    if (n_blocks < 0 || !valid_dtype(ydtype))
        return -1;
    for (int64_t k = 0; k < n_blocks; ++k) {
        const uint8_t *blk = blocks + 144 * k;
        float d = half_at(blk), dmin = half_at(blk + 2);
        const uint8_t *scales = blk + 4, *qs = blk + 16;
        /* 4 groups of 64 elements: 32 bytes of qs each; low nibbles form
         * sub-block 2g, high nibbles sub-block 2g + 1 */
        for (int g = 0; g < 4; ++g) {
            for (int h = 0; h < 2; ++h) {
                int sci, mni;
                q4k_scale_min(scales, 2 * g + h, &sci, &mni);
                float a = d * (float)sci, b = dmin * (float)mni;
                for (int l = 0; l < 32; ++l) {
                    int q = h ? (qs[32 * g + l] >> 4) : (qs[32 * g + l] & 15);
                    store_elem(y, ydtype, 256 * k + 64 * g + 32 * h + l, a * (float)q - b);
                }
            }
        }
    }
    return 0;
}

int bqo_dequant_q6_k(const uint8_t *blocks, int64_t n_blocks, void *y, int ydtype)
{
    if (n_blocks < 0 || !valid_dtype(ydtype))
        return -1;
    for (int64_t k = 0; k < n_blocks; ++k) {
        const uint8_t *blk = blocks + 210 * k;
        const uint8_t *ql = blk, *qh = blk + 128;
        const int8_t *sc = (const int8_t *)(blk + 192);
        float d = half_at(blk + 208);
        /* two halves of 128; in a half, element 32 * c + l (c = 0..3, l < 32)
         * takes its low 4 bits from ql[l + 32 * (c & 1)] (low nibble for c < 2,
         * high nibble otherwise), its top 2 bits from bits 2c, 2c+1 of qh[l],
         * and scale sc[l / 16 + 2 * c] */
        for (int n = 0; n < 2; ++n) {
            for (int c = 0; c < 4; ++c) {
                for (int l = 0; l < 32; ++l) {
                    int lo4 = ql[64 * n + l + 32 * (c & 1)];
                    lo4 = c < 2 ? (lo4 & 15) : (lo4 >> 4);
                    int hi2 = (qh[32 * n + l] >> (2 * c)) & 3;
                    int q = (lo4 | (hi2 << 4)) - 32;
                    float a = d * (float)sc[8 * n + l / 16 + 2 * c];
                    store_elem(y, ydtype, 256 * k + 128 * n + 32 * c + l, a * (float)q);
                }
            }
        }
    }
    return 0;
}

/* Q2_K: sub-block j covers outputs 16j .. 16j + 15.  In half n (outputs
 * 128n ..), output 32c + 16h + l (c < 4, h < 2, l < 16) takes bits 2c, 2c+1
 * of qs[32n + 16h + l]; its sub-block is 8n + 2c + h. */
int bqo_dequant_q2_k(const uint8_t *blocks, int64_t n_blocks, void *y, int ydtype)
{
    if (n_blocks < 0 || !valid_dtype(ydtype))
        return -1;
    for (int64_t k = 0; k < n_blocks; ++k) {
        const uint8_t *blk = blocks + 84 * k;
        const uint8_t *scales = blk, *qs = blk + 16;
        float d = half_at(blk + 80), dmin = half_at(blk + 82);
        for (int n = 0; n < 2; ++n)
            for (int c = 0; c < 4; ++c)
                for (int h = 0; h < 2; ++h) {
                    int j = 8 * n + 2 * c + h;
                    float a = d * (float)(scales[j] & 15), b = dmin * (float)(scales[j] >> 4);
                    for (int l = 0; l < 16; ++l) {
                        int q = (qs[32 * n + 16 * h + l] >> (2 * c)) & 3;
                        store_elem(y, ydtype, 256 * k + 128 * n + 32 * c + 16 * h + l,
                                   a * (float)q - b);
                    }
                }
    }
    return 0;
}

/* Q3_K scale of sub-block i (0..15) from the 12 packed bytes: low 4 bits
 * from byte i (i < 8) or the high nibble of byte i - 8, top 2 bits from
 * byte 8 + i % 4 at bit 2 * (i / 4); stored with an offset of 32. */
static int q3k_scale(const uint8_t *sc, int i)
{
    int lo = i < 8 ? (sc[i] & 15) : (sc[i - 8] >> 4);
    int hi = (sc[8 + (i & 3)] >> (2 * (i >> 2))) & 3;
    return (lo | (hi << 4)) - 32;
}

/* Q3_K: output 128n + 32c + 16h + l takes bits 2c, 2c+1 of qs[32n + 16h + l]
 * and bit 4n + c of hmask[16h + l]; q = low bits - (hmask bit ? 0 : 4). */
int bqo_dequant_q3_k(const uint8_t *blocks, int64_t n_blocks, void *y, int ydtype)
{
    if (n_blocks < 0 || !valid_dtype(ydtype))
        return -1;
    for (int64_t k = 0; k < n_blocks; ++k) {
        const uint8_t *blk = blocks + 110 * k;
        const uint8_t *hmask = blk, *qs = blk + 32, *scales = blk + 96;
        float d = half_at(blk + 108);
        for (int n = 0; n < 2; ++n)
            for (int c = 0; c < 4; ++c)
                for (int h = 0; h < 2; ++h) {
                    float a = d * (float)q3k_scale(scales, 8 * n + 2 * c + h);
                    for (int l = 0; l < 16; ++l) {
                        int low = (qs[32 * n + 16 * h + l] >> (2 * c)) & 3;
                        int hb = (hmask[16 * h + l] >> (4 * n + c)) & 1;
                        int q = low - (hb ? 0 : 4);
                        store_elem(y, ydtype, 256 * k + 128 * n + 32 * c + 16 * h + l,
                                   a * (float)q);
                    }
                }
    }
    return 0;
}

/* Q5_K: as Q4_K (group g of 64 reads qs[32g ..], low nibbles for sub-block
 * 2g, high for 2g + 1) plus bit 2g + h of qh[l] as bit 4 of q. */
int bqo_dequant_q5_k(const uint8_t *blocks, int64_t n_blocks, void *y, int ydtype)
{
    if (n_blocks < 0 || !valid_dtype(ydtype))
        return -1;
    for (int64_t k = 0; k < n_blocks; ++k) {
        const uint8_t *blk = blocks + 176 * k;
        float d = half_at(blk), dmin = half_at(blk + 2);
        const uint8_t *scales = blk + 4, *qh = blk + 16, *qs = blk + 48;
        for (int g = 0; g < 4; ++g)
            for (int h = 0; h < 2; ++h) {
                int sci, mni;
                q4k_scale_min(scales, 2 * g + h, &sci, &mni);
                float a = d * (float)sci, b = dmin * (float)mni;
                for (int l = 0; l < 32; ++l) {
                    int nib = h ? (qs[32 * g + l] >> 4) : (qs[32 * g + l] & 15);
                    int q = nib | (((qh[l] >> (2 * g + h)) & 1) << 4);
                    store_elem(y, ydtype, 256 * k + 64 * g + 32 * h + l, a * (float)q - b);
                }
            }
    }
    return 0;
}

int bqo_dequant_bf16(const uint8_t *src, int64_t n, void *y, int ydtype)
{
    if (n < 0 || !valid_dtype(ydtype))
        return -1;
    for (int64_t i = 0; i < n; ++i)
        store_elem(y, ydtype, i, bqo_bf16_to_f32((uint16_t)(src[2 * i] | (src[2 * i + 1] << 8))));
    return 0;
}

/* ------------------------------------------------------- GGUF encoders -- */

static void put_half(uint8_t *p, float v)
{
    uint16_t h = bqo_f32_to_f16(v);
    p[0] = (uint8_t)(h & 0xff);
    p[1] = (uint8_t)(h >> 8);
}

int bqo_quantize_q8_0(const void *x, int dtype, int64_t n, uint8_t *blocks)
{
    if (n < 0 || n % 32 != 0 || !valid_dtype(dtype))
        return -1;
    for (int64_t k = 0; k < n / 32; ++k) {
        float amax = 0.0f;
        for (int j = 0; j < 32; ++j)
            amax = fmaxf(amax, fabsf(load_elem(x, dtype, 32 * k + j)));
        float d = amax / 127.0f;
        float id = (d == 0.0f) ? 0.0f : 1.0f / d;
        uint8_t *blk = blocks + 34 * k;
        put_half(blk, d);
        for (int j = 0; j < 32; ++j) {
            float r = roundf(load_elem(x, dtype, 32 * k + j) * id);
            int q;
            if (r >= 127.0f)
                q = 127;
            else if (r <= -127.0f)
                q = -127;
            else if (r == r)
                q = (int)r;
            else
                q = 0;
            blk[2 + j] = (uint8_t)(int8_t)q;
        }
    }
    return 0;
}

int bqo_quantize_q4_0(const void *x, int dtype, int64_t n, uint8_t *blocks)
{
    if (n < 0 || n % 32 != 0 || !valid_dtype(dtype))
        return -1;
    for (int64_t k = 0; k < n / 32; ++k) {
        /* the element of largest magnitude, first on ties; starting below
         * every magnitude takes element 0 unless it is NaN */
        float amax = -1.0f, m = 0.0f;
        for (int j = 0; j < 32; ++j) {
            float v = load_elem(x, dtype, 32 * k + j);
            if (fabsf(v) > amax) {
                amax = fabsf(v);
                m = v;
            }
        }
        float d = m / -8.0f;
        float id = (d == 0.0f) ? 0.0f : 1.0f / d;
        uint8_t *blk = blocks + 18 * k;
        put_half(blk, d);
        int q[32];
        for (int j = 0; j < 32; ++j) {
            float t = truncf(load_elem(x, dtype, 32 * k + j) * id + 8.5f);
            if (t >= 15.0f)
                q[j] = 15;
            else if (t >= 0.0f)
                q[j] = (int)t;
            else
                q[j] = 0;
        }
        for (int j = 0; j < 16; ++j)
            blk[2 + j] = (uint8_t)(q[j] | (q[j + 16] << 4));
    }
    return 0;
}
