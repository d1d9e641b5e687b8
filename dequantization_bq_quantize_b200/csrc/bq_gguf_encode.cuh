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
// Kernel design (mirror of the decoder).  A warp step covers 32 blocks (1024
// inputs).  A lane owns 8 consecutive inputs of one block (lanes 4b..4b+3
// share block b), loads them with one or two 16-byte loads - all of a step's
// loads are issued before any is used, kept as raw bits until their turn -
// and the 4 lanes of a block combine
// their maxima with two xor-shuffles.  The lanes write their block's bytes
// into the warp's shared staging buffer, and the warp then stores the step's
// 1088 or 576 bytes (whole 16-byte chunks) with 16-byte stores.  Unaligned
// streams and the last partial step are written byte by byte.
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

// The raw bits of 8 consecutive inputs starting at element e0 (a multiple of
// 8): one 16-byte word for 16-bit types, two for fp32.  Kept raw until use,
// so that a step's loads can all be in flight at once in few registers.
template <int IT> struct Raw8 { uint4 w[IT == kF32 ? 2 : 1]; };

template <int IT>
__device__ __forceinline__ Raw8<IT> load_raw8(const void* x, int64_t e0, bool vec) {
  Raw8<IT> r;
  if constexpr (IT == kF32) {
    const uint32_t* s = static_cast<const uint32_t*>(x) + e0;
    if (vec) {
      r.w[0] = __ldg(reinterpret_cast<const uint4*>(s));
      r.w[1] = __ldg(reinterpret_cast<const uint4*>(s) + 1);
    } else {
      r.w[0] = make_uint4(s[0], s[1], s[2], s[3]);
      r.w[1] = make_uint4(s[4], s[5], s[6], s[7]);
    }
  } else {
    const uint16_t* s = static_cast<const uint16_t*>(x) + e0;
    if (vec) {
      r.w[0] = __ldg(reinterpret_cast<const uint4*>(s));
    } else {
      r.w[0] = make_uint4(s[0] | (uint32_t{s[1]} << 16), s[2] | (uint32_t{s[3]} << 16),
                          s[4] | (uint32_t{s[5]} << 16), s[6] | (uint32_t{s[7]} << 16));
    }
  }
  return r;
}

template <int IT>
__device__ __forceinline__ void widen8(const Raw8<IT>& r, float (&v)[8]) {
  if constexpr (IT == kF32) {
    v[0] = __uint_as_float(r.w[0].x); v[1] = __uint_as_float(r.w[0].y);
    v[2] = __uint_as_float(r.w[0].z); v[3] = __uint_as_float(r.w[0].w);
    v[4] = __uint_as_float(r.w[1].x); v[5] = __uint_as_float(r.w[1].y);
    v[6] = __uint_as_float(r.w[1].z); v[7] = __uint_as_float(r.w[1].w);
  } else {
    const uint32_t w[4] = {r.w[0].x, r.w[0].y, r.w[0].z, r.w[0].w};
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      v[2 * k] = widen_pair_elem<IT>(w[k], 0);
      v[2 * k + 1] = widen_pair_elem<IT>(w[k], 1);
    }
  }
}

__device__ __forceinline__ void store_u16x4(uint8_t* p, uint32_t w0, uint32_t w1) {
  uint16_t* h = reinterpret_cast<uint16_t*>(p);  // 2-byte aligned
  h[0] = static_cast<uint16_t>(w0);
  h[1] = static_cast<uint16_t>(w0 >> 16);
  h[2] = static_cast<uint16_t>(w1);
  h[3] = static_cast<uint16_t>(w1 >> 16);
}

__device__ __forceinline__ uint16_t half_bits(float d) {
  return __half_as_ushort(__float2half_rn(d));
}

// Encode the 8 inputs v of part `part` (inputs 8*part ..) of the block whose
// staging bytes start at bp.  All 32 lanes of the warp must call this
// together (it shuffles); `live` is false for lanes past the last block.
template <int KIND>
__device__ __forceinline__ void gguf_encode8(uint8_t* bp, int part, const float (&v)[8],
                                             bool live) {
  if constexpr (KIND == kQ8_0) {
    float a = 0.0f;
#pragma unroll
    for (int k = 0; k < 8; ++k) a = fmaxf(a, fabsf(v[k]));
    a = fmaxf(a, __shfl_xor_sync(0xffffffffu, a, 1));
    a = fmaxf(a, __shfl_xor_sync(0xffffffffu, a, 2));
    const float d = a / 127.0f;
    const float id = d == 0.0f ? 0.0f : 1.0f / d;
    uint32_t w[2] = {0u, 0u};
#pragma unroll
    for (int k = 0; k < 8; ++k) {
      const float r = roundf(__fmul_rn(v[k], id));
      int q;
      if (r >= 127.0f) q = 127;
      else if (r <= -127.0f) q = -127;
      else if (r == r) q = __float2int_rz(r);
      else q = 0;
      w[k >> 2] |= (static_cast<uint32_t>(q) & 0xFFu) << (8 * (k & 3));
    }
    if (live) {
      store_u16x4(bp + 2 + 8 * part, w[0], w[1]);
      if (part == 0) *reinterpret_cast<uint16_t*>(bp) = half_bits(d);
    }
  } else {  // kQ4_0
    // key: |x| bits above, then (31 - index) and the sign bit: the largest
    // key is the largest magnitude, the lowest index on ties; NaN keys are 0
    uint64_t best = 0;
#pragma unroll
    for (int k = 0; k < 8; ++k) {
      const uint32_t u = __float_as_uint(v[k]);
      const uint32_t mag = u & 0x7FFFFFFFu;
      const uint64_t key =
          mag > 0x7F800000u ? 0ull
                            : (static_cast<uint64_t>(mag) << 32) |
                                  (static_cast<uint32_t>(31 - (8 * part + k)) << 1) | (u >> 31);
      best = key > best ? key : best;
    }
    uint64_t o = __shfl_xor_sync(0xffffffffu, best, 1);
    best = o > best ? o : best;
    o = __shfl_xor_sync(0xffffffffu, best, 2);
    best = o > best ? o : best;
    const float m = __uint_as_float(static_cast<uint32_t>(best >> 32) |
                                    (static_cast<uint32_t>(best & 1u) << 31));
    const float d = m / -8.0f;
    const float id = d == 0.0f ? 0.0f : 1.0f / d;
    uint32_t w[2] = {0u, 0u};
#pragma unroll
    for (int k = 0; k < 8; ++k) {
      const float t = truncf(__fadd_rn(__fmul_rn(v[k], id), 8.5f));
      const uint32_t q = t >= 15.0f ? 15u : (t >= 0.0f ? static_cast<uint32_t>(__float2int_rz(t)) : 0u);
      w[k >> 2] |= q << (8 * (k & 3));
    }
    // parts 2, 3 hold inputs 16..31: their codes become the high nibbles of
    // the bytes that parts 0, 1 hold
    const uint32_t h0 = __shfl_down_sync(0xffffffffu, w[0], 2);
    const uint32_t h1 = __shfl_down_sync(0xffffffffu, w[1], 2);
    if (live && part < 2) {
      store_u16x4(bp + 2 + 8 * part, w[0] | (h0 << 4), w[1] | (h1 << 4));
      if (part == 0) *reinterpret_cast<uint16_t*>(bp) = half_bits(d);
    }
  }
}

template <int KIND, int IT>
__global__ void __launch_bounds__(kGThreads) gguf_encode_kernel(const GEParams p) {
  constexpr int BB = GTraits<KIND>::BB;
  constexpr int STEP_BLOCKS = 32;
  constexpr int STEP_BYTES = STEP_BLOCKS * BB;  // 1088 or 576: whole 16-byte chunks
  constexpr int STEP_CHUNKS = STEP_BYTES / 16;
  constexpr int UNROLL = 4;                     // 8 blocks per warp pass
  static_assert(STEP_BYTES % 16 == 0, "a step must be whole 16-byte chunks");
  __shared__ __align__(16) uint8_t buf[kGThreads / 32][STEP_BYTES];

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  uint8_t* wb = buf[warp];
  const int64_t nsteps = (p.n_blocks + STEP_BLOCKS - 1) / STEP_BLOCKS;
  const int64_t nwarps = static_cast<int64_t>(gridDim.x) * (kGThreads / 32);
  const int part = lane & 3;
  pdl_release();
  pdl_wait();  // x may be written by the previous kernel

  for (int64_t g = static_cast<int64_t>(blockIdx.x) * (kGThreads / 32) + warp; g < nsteps;
       g += nwarps) {
    const int64_t blk0 = g * STEP_BLOCKS;
    const int nblk = static_cast<int>(min(static_cast<int64_t>(STEP_BLOCKS), p.n_blocks - blk0));
    Raw8<IT> raw[UNROLL];
#pragma unroll
    for (int u = 0; u < UNROLL; ++u) {
      const int bl = u * 8 + (lane >> 2);
      if (bl < nblk) {
        raw[u] = load_raw8<IT>(p.x, (blk0 + bl) * 32 + 8 * part, p.vec != 0);
      } else {
#pragma unroll
        for (int i = 0; i < (IT == kF32 ? 2 : 1); ++i) raw[u].w[i] = make_uint4(0u, 0u, 0u, 0u);
      }
    }
#pragma unroll
    for (int u = 0; u < UNROLL; ++u) {
      const int bl = u * 8 + (lane >> 2);
      float v[8];
      widen8<IT>(raw[u], v);
      gguf_encode8<KIND>(wb + bl * BB, part, v, bl < nblk);
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
  }
}

}  // namespace bq
