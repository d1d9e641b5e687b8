/*
 * bq.h - blockwise codebook quantization / dequantization (plain and with
 * compressed statistics), GGUF block dequantization (Q8_0, Q4_0, Q4_1, Q5_0,
 * Q5_1, Q2_K, Q3_K, Q4_K, Q5_K, Q6_K, BF16), GGUF Q8_0 / Q4_0 encoding and a
 * two-stream host-input quantization pipeline on NVIDIA B200 (sm_100a).
 * C ABI of libbq.so.
 *
 * Common contract of every compute entry point
 * -------------------------------------------
 *  - All data pointers are DEVICE pointers on the current CUDA device, owned
 *    and allocated by the caller.  The library allocates nothing, copies
 *    nothing from the host, and never synchronizes.
 *  - All work is enqueued on `stream`, which may be the legacy default stream
 *    (0) if the caller passes it; nothing is ever launched on any other
 *    stream.  This is the stream contract of "bitsandbytes PR #2052, Respect
 *    the current CUDA stream in blockwise quantization" (Summary: launches on
 *    the legacy default stream raced producers on PyTorch's current stream).
 *    Inputs must stay valid and unmodified until the stream work completes.
 *  - Arguments are validated on the host before anything is launched; a bad
 *    argument returns BQ_ERR_INVALID_ARG (or BQ_ERR_UNSUPPORTED) and leaves
 *    every buffer untouched.  n == 0 (or n_blocks == 0) returns BQ_OK with no
 *    launch.  A failed launch returns BQ_ERR_CUDA; bq_last_cuda_error() then
 *    gives the CUDA message (per calling thread).  Faults during execution
 *    surface at the caller's next synchronization, as with any CUDA work.
 *  - Any pointer alignment allowed by the element type is accepted.  16-byte
 *    aligned buffers take the vectorised / TMA path; others a scalar path with
 *    identical results.
 *  - Thread safety: entry points may be called concurrently from several host
 *    threads (no shared host state besides the per-thread error text).
 */
#ifndef BQ_H
#define BQ_H

#include <stddef.h>
#include <stdint.h>
#include <cuda_runtime_api.h>

#ifdef __cplusplus
extern "C" {
#endif

#define BQ_ABI_VERSION 1

#if defined(__GNUC__)
#define BQ_API __attribute__((visibility("default")))
#else
#define BQ_API
#endif

typedef enum bq_status {
    BQ_OK = 0,
    BQ_ERR_INVALID_ARG = 1,   /* bad size, pointer, blocksize or codebook length */
    BQ_ERR_UNSUPPORTED = 2,   /* valid request this library does not implement   */
    BQ_ERR_CUDA = 3           /* a CUDA call failed; see bq_last_cuda_error()    */
} bq_status;

/* Element types of inputs (quantize) and outputs (dequantize). */
typedef enum bq_dtype {
    BQ_F32 = 0,               /* IEEE binary32                    */
    BQ_F16 = 1,               /* IEEE binary16                    */
    BQ_BF16 = 2               /* bfloat16 (top half of a binary32) */
} bq_dtype;

/*
 * Blockwise absmax codebook quantization.
 * Defined by "bitsandbytes PR #2052" (Summary: General8, FP4 and NF4 blockwise
 * quantization; Correctness: FP16/BF16/FP32 inputs, every block size from 32
 * through 4096, full blocks and tails).
 *
 * For block b = elements [b*blocksize, min(n, (b+1)*blocksize)):
 *   absmax[b] = max |x_i|                          (fp32; +0 for an all-zero block)
 *   xn_i      = absmax[b] == 0 ? 0 : x_i / absmax[b]   (fp32, IEEE division)
 *   idx_i     = argmin_j |RN(xn_i - code[j])|      (fp32; lowest j on ties)
 *
 *   x            device, n elements of x_dtype, contiguous.
 *   n            element count, >= 0.
 *   blocksize    power of two in [32, 4096].
 *   code         device, code_entries fp32 values sorted ascending (non-decreasing);
 *                finite.  16 entries -> 4-bit codes, 256 entries -> 8-bit codes.
 *                Unsorted tables are accepted and still give the exact result,
 *                on a slow path (sortedness is checked on the device).
 *   absmax       device, ceil(n / blocksize) fp32, written.
 *   out          device, written: 16 entries: ceil(n/2) bytes, element 2i in the
 *                high nibble of byte i, element 2i+1 in the low nibble (0 if it
 *                does not exist); 256 entries: n bytes, one code per element.
 * Inputs must be finite (non-finite values are outside the contract).
 * Ordering: everything the call reads, `code` included, may be written by
 * any earlier work on `stream`, library calls included.  (The kernel starts
 * under programmatic dependent launch and builds its search tables from
 * `code` while earlier kernels finish; after waiting for them it reads
 * `code` again and rebuilds the tables if any entry changed.)
 */
BQ_API bq_status bq_quantize_blockwise(const void *x, bq_dtype x_dtype, int64_t n,
                                int32_t blocksize, const float *code,
                                int32_t code_entries, float *absmax,
                                uint8_t *out, cudaStream_t stream);

/*
 * Blockwise dequantization, the inverse map of bq_quantize_blockwise:
 *   y_i = narrow_to(y_dtype, RN(code[idx_i] * absmax[i / blocksize]))
 * with one fp32 product and one round-to-nearest-even narrowing.
 *   q        device, packed codes laid out as `out` above.
 *   absmax   device, ceil(n / blocksize) fp32.
 *   code     device, code_entries (16 or 256) fp32 values (any order).
 *   y        device, n elements of y_dtype, written.
 */
BQ_API bq_status bq_dequantize_blockwise(const uint8_t *q, const float *absmax,
                                  int64_t n, int32_t blocksize,
                                  const float *code, int32_t code_entries,
                                  void *y, bq_dtype y_dtype,
                                  cudaStream_t stream);

/*
 * Blockwise quantization with compressed statistics ("bitsandbytes PR #2052",
 * Summary: NF4 storage whose absmax array is itself quantized blockwise with
 * the General8 map).  Two launches on `stream`: the elements as in
 * bq_quantize_blockwise, writing their fp32 statistics to `absmax`, then that
 * array as an fp32 input of nb = ceil(n / blocksize) elements, quantized with
 * `code2` in blocks of `blocksize2`.  No mean is subtracted from the
 * statistics (the page describes none).
 *   code2      device, 256 fp32 entries (the General8 map); code2_entries
 *              must be 256.
 *   blocksize2 power of two in [32, 4096] (256 is the usual choice).
 *   absmax     device, nb fp32, written (the first-level statistics).
 *   absmax2    device, ceil(nb / blocksize2) fp32, written.
 *   qabsmax    device, nb bytes, written (one code2 index per block).
 * Other arguments and errors as bq_quantize_blockwise.
 */
BQ_API bq_status bq_quantize_blockwise_nested(const void *x, bq_dtype x_dtype, int64_t n,
                                  int32_t blocksize, const float *code,
                                  int32_t code_entries, const float *code2,
                                  int32_t code2_entries, int32_t blocksize2,
                                  float *absmax, uint8_t *out, float *absmax2,
                                  uint8_t *qabsmax, cudaStream_t stream);

/*
 * bq_quantize_blockwise_nested for callers that cannot allocate device
 * memory.  (The source pages have no counterpart of this entry point; it
 * exists for the way this library is embedded.)  Some callers cannot call
 * cudaMalloc: for example a plug-in inside a host framework that owns all
 * device memory (a caching allocator, or an arena planned before the run)
 * and hands the plug-in only its inputs and outputs, where an allocation
 * behind the framework's back would break its memory budget and can
 * synchronize the device.  Such a caller usually wants only the compressed
 * statistics, not the fp32 first-level statistics that
 * bq_quantize_blockwise_nested writes to a caller buffer between its two
 * launches.  This entry point keeps that intermediate array in a fixed
 * device array inside the library instead, and otherwise behaves exactly
 * like bq_quantize_blockwise_nested (same arguments without `absmax`, same
 * outputs, bit for bit).
 *
 *  - Size limit: ceil(n / blocksize) <= BQ_NOALLOC_MAX_BLOCKS (2^20 blocks,
 *    4 MiB of fp32), i.e. n <= 2^20 * blocksize.  Larger inputs return
 *    BQ_ERR_INVALID_ARG before anything is launched, and
 *    bq_last_cuda_error() then names the limit.
 *  - Memory: the array is a static device variable of libbq.so, so every
 *    GPU on which the library is used holds those 4 MiB until the process
 *    exits.  The call itself allocates nothing (no cudaMalloc, no
 *    cudaFree, no allocating library routine).
 *  - Set-up: the first call on each device looks up the array's device
 *    address (cudaGetSymbolAddress, with that device current), once.  Make
 *    that first call before any stream capture on the device.
 *  - Sharing: every call on a device uses the same array, and the array
 *    keeps the last call's contents.  Nothing in it needs to start at zero:
 *    each call writes every entry it later reads, in stream order.  Calls
 *    whose work overlaps on the GPU (different streams, or different host
 *    threads, without ordering between them) race on the array and give
 *    wrong results; order them, e.g. by using one stream.
 */
#define BQ_NOALLOC_MAX_BLOCKS (1 << 20)
BQ_API bq_status bq_quantize_blockwise_nested_noalloc(const void *x, bq_dtype x_dtype,
                                  int64_t n, int32_t blocksize, const float *code,
                                  int32_t code_entries, const float *code2,
                                  int32_t code2_entries, int32_t blocksize2,
                                  uint8_t *out, float *absmax2, uint8_t *qabsmax,
                                  cudaStream_t stream);

/*
 * Inverse of bq_quantize_blockwise_nested, in one launch: block b's scale is
 * rebuilt as A_b = RN(code2[qabsmax[b]] * absmax2[b / blocksize2]) - exactly
 * the fp32 value the statistics' own dequantization gives - and then
 * y_i = narrow_to(y_dtype, RN(code[idx_i] * A_(i / blocksize))).  No fp32
 * statistics array is needed.
 */
BQ_API bq_status bq_dequantize_blockwise_nested(const uint8_t *q, const uint8_t *qabsmax,
                                  const float *absmax2, int64_t n, int32_t blocksize,
                                  const float *code, int32_t code_entries,
                                  const float *code2, int32_t code2_entries,
                                  int32_t blocksize2, void *y, bq_dtype y_dtype,
                                  cudaStream_t stream);

/*
 * Quantization of a HOST input, pipelined over two streams ("bitsandbytes PR
 * #2052", B300 measurement: the two-stream pinned host-to-device plus
 * compressed-NF4 pipeline, where each copy and the quantizer that reads it
 * are chained on one stream).  The input is cut into chunks of
 * chunk_elements; chunk i is copied into half (i % 2) of `staging` with
 * cudaMemcpyAsync on stream (i % 2 ? stream1 : stream0) and quantized right
 * after its copy on the same stream (with compressed statistics when code2 is
 * not NULL), so one chunk's copy overlaps the other's quantization.  The
 * outputs are bit-identical to one bq_quantize_blockwise(_nested) call on the
 * whole input.  Ordering: stream1's first copy waits for the work queued on
 * stream0 before the call, and at return stream0 has been made to wait for
 * stream1's work, so the whole call behaves as work on stream0: the outputs
 * are complete in stream0's order.
 * Exception to the common contract: this call reads host memory and creates
 * (and releases) one CUDA event per call.
 *   x_host        host, n elements of x_dtype.  Pinned (page-locked) memory
 *                 gives the overlap; pageable memory works but the copies
 *                 then serialize with the host.  Must stay unchanged until
 *                 stream0's work completes.
 *   code2 ...     NULL for plain statistics (code2_entries, blocksize2,
 *                 absmax2 and qabsmax are then ignored); otherwise as
 *                 bq_quantize_blockwise_nested.
 *   absmax, out   device outputs as bq_quantize_blockwise.
 *   staging       device, 16-byte aligned, staging_bytes >= 2 * chunk_elements
 *                 * element bytes (n * element bytes when n <= chunk_elements).
 *   chunk_elements > 0, a multiple of blocksize (of blocksize * blocksize2
 *                 with compressed statistics).
 *   stream0, stream1  the two streams (may be equal: no overlap then).
 * BQ_ERR_INVALID_ARG for bad sizes, pointers or a staging buffer that is too
 * small; BQ_ERR_CUDA if a copy, launch or the join fails.
 */
BQ_API bq_status bq_quantize_blockwise_host(const void *x_host, bq_dtype x_dtype, int64_t n,
                                  int32_t blocksize, const float *code,
                                  int32_t code_entries, const float *code2,
                                  int32_t code2_entries, int32_t blocksize2,
                                  float *absmax, uint8_t *out, float *absmax2,
                                  uint8_t *qabsmax, void *staging, int64_t staging_bytes,
                                  int64_t chunk_elements, cudaStream_t stream0,
                                  cudaStream_t stream1);

/*
 * GGUF Q8_0 dequantization ("ComfyUI-GGUF PR #472, Cache device-side
 * constants in dequant kernels", Verification table, Q8_0 row: the one type
 * with no shift constant).  Block k is 34 bytes: fp16 d (little endian, bytes
 * 0..1) then 32 signed bytes q_j.  y[32k + j] = narrow_to(y_dtype, d * q_j);
 * the fp32 product is exact.
 *   blocks   device, n_blocks * 34 bytes (any byte alignment).
 *   y        device, 32 * n_blocks elements of y_dtype, written.
 */
BQ_API bq_status bq_dequant_q8_0(const void *blocks, int64_t n_blocks, void *y,
                          bq_dtype y_dtype, cudaStream_t stream);

/*
 * GGUF Q4_0 dequantization (same page, Problem section: each quant byte is
 * split by the shift vector [0, 4], low nibbles first).  Block k is 18 bytes:
 * fp16 d then 16 bytes qs.  For j < 16:
 *   y[32k + j]      = narrow_to(y_dtype, d * ((qs[j] & 15) - 8))
 *   y[32k + 16 + j] = narrow_to(y_dtype, d * ((qs[j] >> 4) - 8))
 *   blocks   device, n_blocks * 18 bytes (any byte alignment).
 *   y        device, 32 * n_blocks elements of y_dtype, written.
 */
BQ_API bq_status bq_dequant_q4_0(const void *blocks, int64_t n_blocks, void *y,
                          bq_dtype y_dtype, cudaStream_t stream);

/*
 * The other block types of the same page's Verification table (Q4_1, Q5_0,
 * Q5_1, Q2_K, Q3_K, Q4_K, Q5_K, Q6_K: 4096 blocks, bf16 target,
 * bit-identical across implementations; BF16 below).  The page names them without spelling out their bytes;
 * these entry points follow the GGUF block layouts below.  All fp16 fields are
 * little endian; every product is exact in fp32, so the output is the
 * correctly rounded value of the formula, the min being added once.
 * Arguments as for bq_dequant_q8_0: blocks are device bytes (any alignment),
 * y receives (elements per block) * n_blocks values of y_dtype.
 *
 * Q4_1: 20-byte blocks {fp16 d, fp16 m, qs[16]}, 32 outputs:
 *   y[32k + j] = d * (qs[j] & 15) + m,  y[32k + 16 + j] = d * (qs[j] >> 4) + m
 */
BQ_API bq_status bq_dequant_q4_1(const void *blocks, int64_t n_blocks, void *y,
                          bq_dtype y_dtype, cudaStream_t stream);

/*
 * Q5_0: 22-byte blocks {fp16 d, uint32 qh, qs[16]}, 32 outputs: output e
 * takes its low 4 bits as in Q4_0 and bit e of qh as bit 4 (q in 0..31):
 *   y[32k + e] = d * (q - 16)
 */
BQ_API bq_status bq_dequant_q5_0(const void *blocks, int64_t n_blocks, void *y,
                          bq_dtype y_dtype, cudaStream_t stream);

/*
 * Q5_1: 24-byte blocks {fp16 d, fp16 m, uint32 qh, qs[16]}, q as in Q5_0:
 *   y[32k + e] = d * q + m
 */
BQ_API bq_status bq_dequant_q5_1(const void *blocks, int64_t n_blocks, void *y,
                          bq_dtype y_dtype, cudaStream_t stream);

/*
 * Q4_K: 144-byte super-blocks {fp16 d, fp16 dmin, scales[12], qs[128]}, 256
 * outputs in 8 sub-blocks of 32.  Sub-block i < 4 has scale scales[i] & 63 and
 * min scales[i + 4] & 63; i >= 4 has scale (scales[i + 4] & 15) |
 * (scales[i - 4] >> 6) << 4 and min (scales[i + 4] >> 4) | (scales[i] >> 6) << 4.
 * Group g (outputs 64g .. 64g + 63) reads qs[32g .. 32g + 31]: low nibbles
 * are sub-block 2g, high nibbles sub-block 2g + 1.
 *   y = d * scale * q - dmin * min
 */
BQ_API bq_status bq_dequant_q4_k(const void *blocks, int64_t n_blocks, void *y,
                          bq_dtype y_dtype, cudaStream_t stream);

/*
 * Q6_K: 210-byte super-blocks {ql[128], qh[64], int8 scales[16], fp16 d}, 256
 * outputs in 16 sub-blocks of 16 (sub-block j uses scales[j]).  In half n
 * (outputs 128n ..), output 32c + l (c < 4, l < 32) takes its low 4 bits from
 * ql[64n + 32(c & 1) + l] (low nibble for c < 2, else high) and bits 4..5
 * from bits 2c, 2c + 1 of qh[32n + l]:
 *   y = d * scales[j] * (q - 32)
 */
BQ_API bq_status bq_dequant_q6_k(const void *blocks, int64_t n_blocks, void *y,
                          bq_dtype y_dtype, cudaStream_t stream);

/*
 * Q2_K: 84-byte super-blocks {scales[16], qs[64], fp16 d, fp16 dmin}, 256
 * outputs in 16 sub-blocks of 16; scales[j] = (min_j << 4) | scale_j.  In
 * half n (outputs 128n ..), output 32c + 16h + l (c < 4, h < 2, l < 16) takes
 * bits 2c, 2c + 1 of qs[32n + 16h + l] and belongs to sub-block 8n + 2c + h:
 *   y = d * scale * q - dmin * min
 */
BQ_API bq_status bq_dequant_q2_k(const void *blocks, int64_t n_blocks, void *y,
                          bq_dtype y_dtype, cudaStream_t stream);

/*
 * Q3_K: 110-byte super-blocks {hmask[32], qs[64], scales[12], fp16 d}, 16
 * sub-blocks of 16 with 6-bit scales s_i: the low 4 bits are byte i (i < 8)
 * or the high nibble of byte i - 8, the top 2 bits come from byte 8 + i % 4
 * at bit 2 * (i / 4).  Output 128n + 32c + 16h + l takes bits 2c, 2c + 1 of
 * qs[32n + 16h + l] as q, minus 4 unless bit 4n + c of hmask[16h + l] is set:
 *   y = d * (s - 32) * q
 */
BQ_API bq_status bq_dequant_q3_k(const void *blocks, int64_t n_blocks, void *y,
                          bq_dtype y_dtype, cudaStream_t stream);

/*
 * Q5_K: 176-byte super-blocks {fp16 d, fp16 dmin, scales[12] packed as Q4_K,
 * qh[32], qs[128]}: as Q4_K, with bit 2g + h of qh[l] (l < 32 the position in
 * the 32-output half) as bit 4 of q:
 *   y = d * scale * q - dmin * min
 */
BQ_API bq_status bq_dequant_q5_k(const void *blocks, int64_t n_blocks, void *y,
                          bq_dtype y_dtype, cudaStream_t stream);

/*
 * BF16 tensor data (the BF16 row of the same table): n little-endian
 * bfloat16 values widened exactly to fp32 and narrowed to y_dtype (a copy for
 * BQ_BF16).  x must be 2-byte aligned; n counts values, not blocks.  NaN
 * payloads are outside the contract (a bf16 output copies them; other
 * outputs give the conversion's NaN).
 */
BQ_API bq_status bq_dequant_bf16(const void *x, int64_t n, void *y, bq_dtype y_dtype,
                          cudaStream_t stream);

/*
 * GGUF Q8_0 / Q4_0 encoders: the inverse direction of bq_dequant_q8_0 and
 * bq_dequant_q4_0 (same page: the Problem section and Verification table
 * give the block formats, not an encoder).  They follow the GGUF format's
 * reference quantizer, in fp32 on the exactly widened input:
 *   Q8_0: d = max|x| / 127, id = (d == 0 ? 0 : 1/d),
 *         q_j = round-half-away(x_j * id); block = fp16(d), int8 q[32]
 *   Q4_0: m = the element of largest |x| (the first on ties), d = m / -8,
 *         id = (d == 0 ? 0 : 1/d), q_j = min(15, trunc(x_j * id + 8.5));
 *         block = fp16(d), byte j = q_j | q_(j+16) << 4
 * fp16(d) rounds to nearest even.  Non-finite inputs are clamped (Q8_0 to
 * [-127, 127], Q4_0 to [0, 15], NaN to 0; NaN never chosen as m), so every
 * input gives defined bytes.
 *   x        device, n elements of x_dtype (aligned to the element size);
 *            n must be a multiple of 32 (GGUF rows are whole blocks).
 *   blocks   device, (n / 32) * 34 (Q8_0) or * 18 (Q4_0) bytes, written
 *            (any byte alignment).
 * BQ_ERR_INVALID_ARG for n < 0, n % 32 != 0, a bad dtype, null or misaligned
 * pointers; n == 0 returns BQ_OK without a launch.
 */
BQ_API bq_status bq_quantize_q8_0(const void *x, bq_dtype x_dtype, int64_t n, void *blocks,
                                  cudaStream_t stream);
BQ_API bq_status bq_quantize_q4_0(const void *x, bq_dtype x_dtype, int64_t n, void *blocks,
                                  cudaStream_t stream);

/* Static text for a status code. */
BQ_API const char *bq_status_string(bq_status s);

/* Text of the last CUDA error seen by an entry point on this host thread
 * ("" if none).  The pointer stays valid until the next call on this thread. */
BQ_API const char *bq_last_cuda_error(void);

/*
 * Device-side fault word.  Kernels that wait on an mbarrier give up after a
 * bounded time instead of hanging, set a bit here and return; results of that
 * launch are then invalid.  Reads the word of the current device (this call
 * SYNCHRONIZES the device), stores it in *fault and, if reset != 0, clears it.
 * 0 means no fault was recorded.  Bits: 1 / 2 quantize consumer / producer
 * wait, 4 / 8 dequantize consumer / producer wait.
 */
BQ_API bq_status bq_device_fault(uint32_t *fault, int32_t reset);

/* BQ_ABI_VERSION of the loaded library. */
BQ_API int32_t bq_abi_version(void);

#ifdef __cplusplus
}
#endif
#endif /* BQ_H */
