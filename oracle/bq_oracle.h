/*
 * bq_oracle.h - plain, slow, single-threaded CPU reference for blockwise
 * codebook quantization / dequantization and GGUF block dequantization
 * (Q8_0, Q4_0, Q4_1, Q5_0, Q5_1, Q2_K, Q3_K, Q4_K, Q5_K, Q6_K, BF16).
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing in the library path may include, link
 * or call this code: only the tests, the package's smoke check and the
 * benchmark's CPU-baseline leg use it.  It shares no code, header, table or
 * constant with the CUDA implementation.
 *
 * What it follows (page titles of the source material):
 *  - "bitsandbytes PR #2052, Respect the current CUDA stream in blockwise
 *    quantization", Summary and Correctness sections: blockwise quantization
 *    with General8 (dynamic 8-bit), FP4 and NF4 maps, block sizes 32..4096,
 *    full blocks and tails, FP16/BF16/FP32 inputs.
 *  - "ComfyUI-GGUF PR #472, Cache device-side constants in dequant kernels",
 *    Problem section (Q4_0 low nibble then high nibble, shift vector [0, 4])
 *    and the Verification table (Q8_0 and Q4_0 rows).
 *  - The same page's Verification table also lists Q4_1, Q5_0, Q5_1, Q2_K,
 *    Q3_K, Q4_K, Q5_K, Q6_K and BF16 (4096 blocks, bf16 target,
 *    bit-identical).  The pages do not
 *    spell out those block layouts; the functions below follow the GGUF
 *    format's published block layouts, and the tests pin them against the
 *    gguf package's own dequantizer and hand-worked blocks.
 *  - "Model-Optimizer PR #2448" review notes: lowest index wins on equal
 *    error; fused multiply-add changes near-ties, so this file is compiled
 *    with contraction off (-ffp-contract=off) and no fast-math.
 *
 * Every floating-point operation here is one IEEE-754 binary32 operation
 * rounded to nearest-even, in source order.
 */
#ifndef BQ_ORACLE_H
#define BQ_ORACLE_H

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Element type codes used by this oracle (its own numbering). */
enum { BQO_F32 = 0, BQO_F16 = 1, BQO_BF16 = 2 };

/* Exact widening and round-to-nearest-even narrowing. */
float    bqo_f16_to_f32(uint16_t h);
float    bqo_bf16_to_f32(uint16_t h);
uint16_t bqo_f32_to_f16(float f);
uint16_t bqo_f32_to_bf16(float f);

/* Nearest codebook entry: argmin_j |RN(xn - code[j])|, lowest j on ties. */
int bqo_nearest_code(float xn, const float *code, int entries);

/*
 * Blockwise absmax codebook quantization of x[0..n) (element type dtype).
 * absmax[b] = max |x_i| over block b (the last block may be short).
 * entries == 16: out has ceil(n/2) bytes, element 2i in the high nibble of
 * byte i, element 2i+1 in the low nibble (0 when it does not exist).
 * entries == 256: out has n bytes, one code per element.
 * Returns 0 on success, -1 on a bad argument.
 */
int bqo_quantize_blockwise(const void *x, int dtype, int64_t n, int blocksize,
                           const float *code, int entries,
                           float *absmax, uint8_t *out);

/* y_i = narrow(RN(code[idx_i] * absmax[i / blocksize])). */
int bqo_dequantize_blockwise(const uint8_t *q, const float *absmax, int64_t n,
                             int blocksize, const float *code, int entries,
                             void *y, int ydtype);

/* GGUF Q8_0: 34-byte blocks {fp16 d (little endian), int8 q[32]}. */
int bqo_dequant_q8_0(const uint8_t *blocks, int64_t n_blocks, void *y, int ydtype);

/* GGUF Q4_0: 18-byte blocks {fp16 d, uint8 qs[16]};
 * y[32k+j] = d*((qs[j] & 15) - 8), y[32k+16+j] = d*((qs[j] >> 4) - 8). */
int bqo_dequant_q4_0(const uint8_t *blocks, int64_t n_blocks, void *y, int ydtype);

/* GGUF Q4_1: 20-byte blocks {fp16 d, fp16 m, uint8 qs[16]};
 * y[32k+j] = d*(qs[j] & 15) + m, y[32k+16+j] = d*(qs[j] >> 4) + m. */
int bqo_dequant_q4_1(const uint8_t *blocks, int64_t n_blocks, void *y, int ydtype);

/* GGUF Q5_0: 22-byte blocks {fp16 d, uint32 qh (little endian), uint8 qs[16]};
 * element e's 5-bit value is its nibble (as Q4_0) plus bit e of qh as bit 4;
 * y = d*(value - 16). */
int bqo_dequant_q5_0(const uint8_t *blocks, int64_t n_blocks, void *y, int ydtype);

/* GGUF Q5_1: 24-byte blocks {fp16 d, fp16 m, uint32 qh, uint8 qs[16]};
 * y = d*value + m. */
int bqo_dequant_q5_1(const uint8_t *blocks, int64_t n_blocks, void *y, int ydtype);

/* GGUF Q4_K: 144-byte super-blocks of 256 {fp16 d, fp16 dmin, uint8 scales[12],
 * uint8 qs[128]}: 8 sub-blocks of 32 with 6-bit scales sc[i] and mins mn[i];
 * y = d*sc*q - dmin*mn with q the 4-bit value. */
int bqo_dequant_q4_k(const uint8_t *blocks, int64_t n_blocks, void *y, int ydtype);

/* GGUF Q6_K: 210-byte super-blocks of 256 {uint8 ql[128], uint8 qh[64],
 * int8 scales[16], fp16 d}: 16 sub-blocks of 16, y = d*scale*(q - 32) with q
 * the 6-bit value (4 low bits from ql, 2 high bits from qh). */
int bqo_dequant_q6_k(const uint8_t *blocks, int64_t n_blocks, void *y, int ydtype);

/* GGUF Q2_K: 84-byte super-blocks of 256 {uint8 scales[16], uint8 qs[64],
 * fp16 d, fp16 dmin}: 16 sub-blocks of 16, scale byte j = (min << 4) | scale;
 * y = d*scale*q - dmin*min with q the 2-bit value. */
int bqo_dequant_q2_k(const uint8_t *blocks, int64_t n_blocks, void *y, int ydtype);

/* GGUF Q3_K: 110-byte super-blocks of 256 {uint8 hmask[32], uint8 qs[64],
 * uint8 scales[12], fp16 d}: 16 sub-blocks of 16 with 6-bit scales s
 * (value s - 32); q = 2 low bits from qs, minus 4 when the hmask bit is 0;
 * y = d*(s - 32)*q. */
int bqo_dequant_q3_k(const uint8_t *blocks, int64_t n_blocks, void *y, int ydtype);

/* GGUF Q5_K: 176-byte super-blocks of 256 {fp16 d, fp16 dmin, uint8
 * scales[12] (packed as Q4_K), uint8 qh[32], uint8 qs[128]}: as Q4_K with a
 * fifth bit from qh; y = d*sc*q - dmin*mn. */
int bqo_dequant_q5_k(const uint8_t *blocks, int64_t n_blocks, void *y, int ydtype);

/* GGUF BF16: n raw bfloat16 values (little endian) widened exactly, then
 * narrowed to ydtype. */
int bqo_dequant_bf16(const uint8_t *src, int64_t n, void *y, int ydtype);

/*
 * GGUF encoders (the inverse direction of Q8_0 / Q4_0), following the GGUF
 * format's reference quantizer.  x holds n elements (n a multiple of 32) of
 * element type dtype; blocks receives n / 32 blocks.  All arithmetic is fp32
 * on the exactly widened input.
 *
 * Q8_0: amax = max |x| over the block (NaN ignored), d = amax / 127,
 * id = (d == 0 ? 0 : 1 / d), q_j = round-half-away(x_j * id), then clamped
 * to [-127, 127] (only non-finite values reach the clamp; NaN gives 0);
 * the block stores fp16(d) (round to nearest even) and the q_j as int8.
 *
 * Q4_0: m = the element of largest |x| (the first one on ties, NaN never
 * chosen, +0 if every element is NaN), d = m / -8, id = (d == 0 ? 0 : 1 / d),
 * t_j = trunc(x_j * id + 8.5), q_j = 15 if t_j >= 15, else t_j if t_j >= 0,
 * else 0 (NaN gives 0); byte j = q_j | q_(j+16) << 4; the block stores fp16(d).
 * Returns 0, or -1 on a bad argument.
 */
int bqo_quantize_q8_0(const void *x, int dtype, int64_t n, uint8_t *blocks);
int bqo_quantize_q4_0(const void *x, int dtype, int64_t n, uint8_t *blocks);

#ifdef __cplusplus
}
#endif
#endif
