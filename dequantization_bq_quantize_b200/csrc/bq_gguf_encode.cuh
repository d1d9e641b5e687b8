// bq_gguf_encode.cuh - GGUF Q8_0 / Q4_0 encoders (sm_100a): the inverse of the
// Q8_0 and Q4_0 block formats of "ComfyUI-GGUF PR #472, Cache device-side
// constants in dequant kernels" (Problem section and Verification table).
// The page gives the formats but no encoder; this follows the GGUF format's
// reference quantizer, all in fp32 on the exactly widened input:
//   Q8_0: amax = max |x| (NaN ignored), d = amax / 127, id = d ? 1/d : 0,
//         q = round-half-away(x * id), clamped to [-127, 127] (NaN -> 0);
//         block = fp16(d), 32 int8 q
//   Q4_0: m = the element of largest |x|, the first on ties (NaN never
//         chosen; +0 when every element is NaN), d = m / -8, id = d ? 1/d : 0,
//         t = trunc(x * id + 8.5), q = 15 if t >= 15, t if t >= 0, else 0;
//         block = fp16(d), byte j = q_j | q_(j+16) << 4
// The divisions are IEEE (the library is built with -prec-div=true), the
// products and the add are single roundings (-fmad=false), so the bytes are
// exactly the reference quantizer's.  The clamps only act on non-finite
// values, where the reference leaves the integer conversion undefined.
//
// Kernel design.  One lane encodes one whole block, so the two IEEE
// divisions per block are shared by its 32 inputs; a warp step is 32 blocks
// (2 KiB of bf16), loaded one step ahead into registers with 16-byte loads
// and kept as raw bits until used.  Each block first takes a block-uniform
// test: if its magnitudes are finite (a NaN-propagating max finds any NaN or
// infinity) and 1/d is finite, every scaled value lies in [-127.001, 127.001]
// (Q8_0) or x * id + 8.5 in [0.4999, 16.5] (Q4_0), the clamps cannot act, and
// the fast path runs:
//   Q8_0: t = x * id, v = RZ(t + copysign(0.5, t)) (packed, round
//         toward zero), q = trunc(v).  Rounding |t| + 0.5 toward zero never
//         carries it past an integer, so trunc(v) = sign(t) * floor(|t| + 0.5),
//         which is round-half-away(t).
//   Q4_0: v = RN(RN(x * id) + 8.5) (packed add), z = RZ(v + 2^23): for v >= 0 the
//         low mantissa bits of z are floor(v) = trunc(v); the clamp to 15 is an
//         integer min on the bits.  d = m * (-1/8) is the same correctly
//         rounded value as m / -8, since -1/8 is exact.
// The products x * id are scalar __fmul_rn: a packed f32x2 multiply whose
// only use is a packed add can be contracted into one fma by the code
// generator, even with explicit .rn, and that skips the product's rounding
// (seen with bf16 inputs, where x * id + 8.5 lands on integers often).
// Other blocks take the exact scalar path with the clamps.  The lanes stage
// their blocks in the warp's shared buffer with 16-bit stores (a 34- or
// 18-byte block is 2-byte aligned there) and the warp stores the step's 1088
// or 576 bytes with 16-byte stores.  Unaligned streams and the last partial
// step are read element by element and written byte by byte.
#pragma once

#include "bq_common.cuh"
#include "bq_gguf.cuh"

namespace bq {

struct GEParams {
  const void* x;
  uint8_t* blocks;
  int64_t n_blocks;
  int32_t vec;  // x and blocks are 16-byte aligned
};

// The raw bits of one block of 32 inputs: 16 words of two 16-bit elements
// (element 2i in the low half of word i) or 32 fp32 words.
template <int IT> struct RawBlk {
  static constexpr int W = IT == kF32 ? 32 : 16;
  uint32_t w[W];
};

template <int IT>
__device__ __forceinline__ float blk_elem(const RawBlk<IT>& r, int j) {
  if constexpr (IT == kF32) return __uint_as_float(r.w[j]);
  else return widen_pair_elem<IT>(r.w[j >> 1], j & 1);
}

template <int IT>
__device__ __forceinline__ void load_blk(RawBlk<IT>& r, const void* x, int64_t blk, bool vec) {
  constexpr int W = RawBlk<IT>::W;
  if (vec) {
    const uint4* s = reinterpret_cast<const uint4*>(static_cast<const uint8_t*>(x) + blk * (4 * W));
#pragma unroll
    for (int i = 0; i < W / 4; ++i) {
      const uint4 a = __ldg(s + i);
      r.w[4 * i] = a.x; r.w[4 * i + 1] = a.y; r.w[4 * i + 2] = a.z; r.w[4 * i + 3] = a.w;
    }
  } else if constexpr (IT == kF32) {
    const uint32_t* s = static_cast<const uint32_t*>(x) + blk * 32;
#pragma unroll
    for (int j = 0; j < 32; ++j) r.w[j] = s[j];
  } else {
    const uint16_t* s = static_cast<const uint16_t*>(x) + blk * 32;
#pragma unroll
    for (int i = 0; i < 16; ++i) r.w[i] = s[2 * i] | (uint32_t{s[2 * i + 1]} << 16);
  }
}

// max |x| over the block, NaN if any element is NaN
template <int IT>
__device__ __forceinline__ float blk_amax_nan(const RawBlk<IT>& r) {
  if constexpr (IT == kF32) {
    float m[16];
#pragma unroll
    for (int i = 0; i < 16; ++i) m[i] = max_nan(fabsf(blk_elem(r, 2 * i)), fabsf(blk_elem(r, 2 * i + 1)));
#pragma unroll
    for (int s = 8; s >= 1; s >>= 1)
#pragma unroll
      for (int i = 0; i < s; ++i) m[i] = max_nan(m[i], m[i + s]);
    return m[0];
  } else {
    uint32_t m[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) m[i] = amax2<IT>(r.w[2 * i], r.w[2 * i + 1]);
#pragma unroll
    for (int s = 4; s >= 1; s >>= 1)
#pragma unroll
      for (int i = 0; i < s; ++i) m[i] = amax2<IT>(m[i], m[i + s]);
    return max_nan(fabsf(widen_pair_elem<IT>(m[0], 0)), fabsf(widen_pair_elem<IT>(m[0], 1)));
  }
}

__device__ __forceinline__ uint64_t add_rz2(uint64_t a, uint64_t b) {
  uint64_t d;
  asm("add.rz.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
  return d;
}
__device__ __forceinline__ uint64_t add_rn2(uint64_t a, uint64_t b) {
  uint64_t d;
  asm("add.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
  return d;
}

// low bytes of four words -> one word
__device__ __forceinline__ uint32_t low_bytes4(uint32_t a, uint32_t b, uint32_t c, uint32_t d) {
  return __byte_perm(__byte_perm(a, b, 0x0040u), __byte_perm(c, d, 0x0040u), 0x5410u);
}

__device__ __forceinline__ uint16_t half_bits(float d) {
  return __half_as_ushort(__float2half_rn(d));
}

// Q8_0 code of one value, exact reference semantics including the clamps
__device__ __forceinline__ uint32_t q8_exact(float x, float id) {
  const float r = roundf(__fmul_rn(x, id));
  int q;
  if (r >= 127.0f) q = 127;
  else if (r <= -127.0f) q = -127;
  else if (r == r) q = __float2int_rz(r);
  else q = 0;
  return static_cast<uint32_t>(q);
}

// Q4_0 code of one value, exact reference semantics including the clamps
__device__ __forceinline__ uint32_t q4_exact(float x, float id) {
  const float t = truncf(__fadd_rn(__fmul_rn(x, id), 8.5f));
  return t >= 15.0f ? 15u : (t >= 0.0f ? static_cast<uint32_t>(__float2int_rz(t)) : 0u);
}

// Q4_0 from the block's largest magnitude and its first element m: the fast
// path when both are usable, else the exact scalar path with the clamps.
template <int IT>
__device__ __forceinline__ void encode_q4_from_m(const RawBlk<IT>& r, float amax, float m,
                                                 uint32_t& dh, uint32_t (&q)[8]) {
  const float kInf = __int_as_float(0x7f800000);
  const float d = __fmul_rn(m, -0.125f);
  const float id = d == 0.0f ? 0.0f : 1.0f / d;  // of either sign here
  if (amax < kInf && fabsf(id) < kInf) {
    const uint64_t h2 = pack2(8.5f, 8.5f), m2 = pack2(8388608.0f, 8388608.0f);
    uint32_t z[32];
#pragma unroll
    for (int k = 0; k < 16; ++k) {
      // scalar products (never contracted), then packed adds
      const uint64_t t = pack2(__fmul_rn(blk_elem(r, 2 * k), id), __fmul_rn(blk_elem(r, 2 * k + 1), id));
      float z0, z1;
      unpack2(add_rz2(add_rn2(t, h2), m2), z0, z1);  // 2^23 + trunc(x * id + 8.5)
      z[2 * k] = min(__float_as_uint(z0), 0x4B00000Fu);
      z[2 * k + 1] = min(__float_as_uint(z1), 0x4B00000Fu);
    }
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const uint32_t lo = low_bytes4(z[4 * i], z[4 * i + 1], z[4 * i + 2], z[4 * i + 3]);
      const uint32_t hi = low_bytes4(z[16 + 4 * i], z[17 + 4 * i], z[18 + 4 * i], z[19 + 4 * i]);
      q[i] = lo | (hi << 4);  // every byte of lo and hi is at most 15
    }
    dh = half_bits(d);
  } else {
    // the first strictly larger magnitude, starting below every magnitude;
    // NaN never wins.  Magnitudes compare as integers (the order of the
    // absolute bits of non-NaN floats), with NaN excluded explicitly.
    int32_t best = -1;
    float ms = 0.0f;
#pragma unroll
    for (int j = 0; j < 32; ++j) {
      const float v = blk_elem(r, j);
      const int32_t mag = static_cast<int32_t>(__float_as_uint(v) & 0x7FFFFFFFu);
      if (mag <= 0x7F800000 && mag > best) {
        best = mag;
        ms = v;
      }
    }
    const float ds = __fmul_rn(ms, -0.125f);
    const float ids = ds == 0.0f ? 0.0f : 1.0f / ds;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const uint32_t lo = low_bytes4(q4_exact(blk_elem(r, 4 * i), ids),
                                     q4_exact(blk_elem(r, 4 * i + 1), ids),
                                     q4_exact(blk_elem(r, 4 * i + 2), ids),
                                     q4_exact(blk_elem(r, 4 * i + 3), ids));
      const uint32_t hi = low_bytes4(q4_exact(blk_elem(r, 16 + 4 * i), ids),
                                     q4_exact(blk_elem(r, 17 + 4 * i), ids),
                                     q4_exact(blk_elem(r, 18 + 4 * i), ids),
                                     q4_exact(blk_elem(r, 19 + 4 * i), ids));
      q[i] = lo | (hi << 4);
    }
    dh = half_bits(ds);
  }
}

// Encode one block: dh = fp16 bits of d; q = the block's quant bytes
// (8 words for Q8_0, 4 for Q4_0) in memory order.
template <int KIND, int IT>
__device__ __forceinline__ void encode_block(const RawBlk<IT>& r, uint32_t& dh, uint32_t (&q)[8]) {
  const float kInf = __int_as_float(0x7f800000);
  if constexpr (KIND == kQ4_0 && IT != kF32) {
    // 16-bit inputs: packed signed max and min give the largest magnitude
    // and, unless +amax and -amax both occur, the sign of every element that
    // has it - so the first such element is known without a search
    uint32_t mx[8], mn[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      mx[i] = smax2<IT>(r.w[2 * i], r.w[2 * i + 1]);
      mn[i] = smin2<IT>(r.w[2 * i], r.w[2 * i + 1]);
    }
#pragma unroll
    for (int st = 4; st >= 1; st >>= 1)
#pragma unroll
      for (int i = 0; i < st; ++i) {
        mx[i] = smax2<IT>(mx[i], mx[i + st]);
        mn[i] = smin2<IT>(mn[i], mn[i + st]);
      }
    const float hi = max_nan(widen_pair_elem<IT>(mx[0], 0), widen_pair_elem<IT>(mx[0], 1));
    const float lo = min_nan(widen_pair_elem<IT>(mn[0], 0), widen_pair_elem<IT>(mn[0], 1));
    const float amax = max_nan(hi, -lo);  // NaN if the block holds a NaN
    float m;
    if (amax > 0.0f && hi != -lo) {
      m = hi == amax ? hi : lo;
    } else {
      // zero block, a +amax / -amax tie, or NaN: the first element of
      // largest magnitude by a scan (scanning down, the last match wins)
      m = 0.0f;
#pragma unroll
      for (int j = 31; j >= 0; --j) m = fabsf(blk_elem(r, j)) == amax ? blk_elem(r, j) : m;
    }
    encode_q4_from_m(r, amax, m, dh, q);
    return;
  }
  const float amax = blk_amax_nan(r);  // NaN if the block holds a NaN
  if constexpr (KIND == kQ8_0) {
    const float d = amax / 127.0f;
    const float id = d == 0.0f ? 0.0f : 1.0f / d;
    if (amax < kInf && id < kInf) {
      uint32_t b[32];
#pragma unroll
      for (int k = 0; k < 16; ++k) {
        // scalar products: a packed multiply followed by a packed add may be
        // contracted into one fma by the code generator, which would skip
        // the rounding of the product
        const float t0 = __fmul_rn(blk_elem(r, 2 * k), id);
        const float t1 = __fmul_rn(blk_elem(r, 2 * k + 1), id);
        const float c0 = __uint_as_float((__float_as_uint(t0) & 0x80000000u) | 0x3F000000u);
        const float c1 = __uint_as_float((__float_as_uint(t1) & 0x80000000u) | 0x3F000000u);
        float v0, v1;
        unpack2(add_rz2(pack2(t0, t1), pack2(c0, c1)), v0, v1);
        b[2 * k] = static_cast<uint32_t>(__float2int_rz(v0));
        b[2 * k + 1] = static_cast<uint32_t>(__float2int_rz(v1));
      }
#pragma unroll
      for (int i = 0; i < 8; ++i) q[i] = low_bytes4(b[4 * i], b[4 * i + 1], b[4 * i + 2], b[4 * i + 3]);
      dh = half_bits(d);
    } else {
      float a = 0.0f;  // NaN ignored
#pragma unroll
      for (int j = 0; j < 32; ++j) a = fmaxf(a, fabsf(blk_elem(r, j)));
      const float ds = a / 127.0f;
      const float ids = ds == 0.0f ? 0.0f : 1.0f / ds;
#pragma unroll
      for (int i = 0; i < 8; ++i)
        q[i] = low_bytes4(q8_exact(blk_elem(r, 4 * i), ids), q8_exact(blk_elem(r, 4 * i + 1), ids),
                          q8_exact(blk_elem(r, 4 * i + 2), ids), q8_exact(blk_elem(r, 4 * i + 3), ids));
      dh = half_bits(ds);
    }
  } else {  // kQ4_0, fp32 input
    // the first element whose magnitude is amax (scanning down, the last
    // match is the lowest index); meaningful only when amax is finite
    float m = 0.0f;
#pragma unroll
    for (int j = 31; j >= 0; --j) m = fabsf(blk_elem(r, j)) == amax ? blk_elem(r, j) : m;
    encode_q4_from_m(r, amax, m, dh, q);
  }
}

template <int KIND, int IT>
__global__ void __launch_bounds__(kGThreads) gguf_encode_kernel(const GEParams p) {
  constexpr int BB = GTraits<KIND>::BB;
  constexpr int QW = KIND == kQ8_0 ? 8 : 4;      // quant words per block
  constexpr int STEP_BLOCKS = 32;                 // one block per lane
  constexpr int STEP_BYTES = STEP_BLOCKS * BB;    // 1088 or 576: whole 16-byte chunks
  constexpr int STEP_CHUNKS = STEP_BYTES / 16;
  static_assert(STEP_BYTES % 16 == 0, "a step must be whole 16-byte chunks");
  __shared__ __align__(16) uint8_t buf[kGThreads / 32][STEP_BYTES];

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  uint8_t* wb = buf[warp];
  uint16_t* mine = reinterpret_cast<uint16_t*>(wb + lane * BB);  // 2-byte aligned
  const int64_t nsteps = (p.n_blocks + STEP_BLOCKS - 1) / STEP_BLOCKS;
  const int64_t nwarps = static_cast<int64_t>(gridDim.x) * (kGThreads / 32);
  pdl_release();
  pdl_wait();  // x may be written by the previous kernel

  auto fetch = [&](int64_t g, RawBlk<IT>& r) {
    const int64_t blk = g * STEP_BLOCKS + lane;
    if (blk < p.n_blocks) load_blk<IT>(r, p.x, blk, p.vec != 0);
  };
  RawBlk<IT> cur, nxt;
  int64_t g = static_cast<int64_t>(blockIdx.x) * (kGThreads / 32) + warp;
  if (g < nsteps) fetch(g, cur);

  for (; g < nsteps; g += nwarps) {
    if (g + nwarps < nsteps) fetch(g + nwarps, nxt);
    const int64_t blk0 = g * STEP_BLOCKS;
    const int nblk = static_cast<int>(min(static_cast<int64_t>(STEP_BLOCKS), p.n_blocks - blk0));
    if (lane < nblk) {
      uint32_t dh, q[8];
      encode_block<KIND, IT>(cur, dh, q);
      mine[0] = static_cast<uint16_t>(dh);
#pragma unroll
      for (int i = 0; i < QW; ++i) {
        mine[1 + 2 * i] = static_cast<uint16_t>(q[i]);
        mine[2 + 2 * i] = static_cast<uint16_t>(q[i] >> 16);
      }
    }
    __syncwarp();
    uint8_t* dst = p.blocks + blk0 * BB;
    if (p.vec && nblk == STEP_BLOCKS) {
      for (int c = lane; c < STEP_CHUNKS; c += 32)
        reinterpret_cast<uint4*>(dst)[c] = reinterpret_cast<const uint4*>(wb)[c];
    } else {
      for (int i = lane; i < nblk * BB; i += 32) dst[i] = wb[i];
    }
    __syncwarp();
    cur = nxt;
  }
}

}  // namespace bq
