// bq_gguf.cuh - GGUF Q8_0 / Q4_0 dequantization (sm_100a).
//
// Formats ("ComfyUI-GGUF PR #472, Cache device-side constants in dequant
// kernels", Problem section and Verification table):
//   Q8_0 block = fp16 d + 32 signed bytes q:       y = d * q
//   Q4_0 block = fp16 d + 16 bytes qs, shifts [0, 4]: y[j] = d * ((qs[j] & 15) - 8),
//                                                    y[16 + j] = d * ((qs[j] >> 4) - 8)
// The fp32 products are exact (an 11-bit d times |q| <= 128), so the narrowed
// output is the correctly rounded value.  The page's point - no per-call
// host-to-device constants - holds trivially here: the shift and offset live
// in registers.
//
// Kernel design.  A warp takes 4 groups of 8 blocks per step (32 blocks:
// 1088 B for Q8_0, 576 B for Q4_0).  A group of 8 blocks is 272 or 144 bytes,
// a whole number of 16-byte chunks, so in a 16-byte aligned stream every group
// starts aligned and the warp stages its 4 groups into its shared buffer with
// up to three 16-byte loads per lane, fetched into registers one step ahead.  Lane l
// then decodes 8 outputs of block l/4 of each group and writes them as one
// 16-byte store, so each warp store covers 512 contiguous bytes of bf16
// output.  Bytes become floats with the 2^23 trick: a byte b placed in the low
// mantissa bits of 2^23 is the float 2^23 + b, and subtracting 2^23 + offset
// is exact.  Unaligned streams and the last partial step are staged byte by
// byte.
#pragma once

#include "bq_common.cuh"

namespace bq {

enum : int { kQ8_0 = 0, kQ4_0 = 1 };

struct GParams {
  const uint8_t* blocks;
  void* y;
  int64_t n_blocks;
  int32_t vec;   // blocks and y are 16-byte aligned
};

constexpr int kGThreads = 256;
constexpr int kGGroup = 8;   // blocks per group (one warp-wide decode)
constexpr int kGUnroll = 4;  // groups per warp step

template <int KIND> struct GTraits;
template <> struct GTraits<kQ8_0> { static constexpr int BB = 34; };
template <> struct GTraits<kQ4_0> { static constexpr int BB = 18; };

// byte k of w placed in the low mantissa of 2^23: the float 2^23 + byte
__device__ __forceinline__ float byte_as_float(uint32_t w, int k) {
  return __uint_as_float(__byte_perm(w, 0x4B000000u, 0x7540u + k));
}

// Eight bytes starting at any 2-byte aligned shared address: three aligned
// 32-bit loads and a funnel shift by 0 or 16 bits.  Plain C++ loads, so that
// they stay ordered after the warp's staging stores and __syncwarp (the
// address does not depend on the staged data).
__device__ __forceinline__ void load8_at2(const uint8_t* ptr, uint32_t& w0, uint32_t& w1) {
  const uintptr_t a = reinterpret_cast<uintptr_t>(ptr);
  const uint32_t* wp = reinterpret_cast<const uint32_t*>(a & ~static_cast<uintptr_t>(3));
  const uint32_t sh = static_cast<uint32_t>(a & 3u) * 8u;
  const uint32_t x0 = wp[0], x1 = wp[1], x2 = wp[2];
  w0 = __funnelshift_r(x0, x1, sh);
  w1 = __funnelshift_r(x1, x2, sh);
}

// Decode 8 outputs (part `part` of the block at bp) to narrowed words:
// v = (float(2^23 + byte) - (2^23 + offset)) * d, two lanes per packed op.
template <int KIND, int OT>
__device__ __forceinline__ void gguf_decode8(const uint8_t* bp, int part, float (&v)[8]) {
  const float d = __half2float(*reinterpret_cast<const __half*>(bp));
  uint32_t w0, w1;
  load8_at2(bp + 2 + (KIND == kQ8_0 ? 8 * part : 8 * (part & 1)), w0, w1);
  float off;
  if constexpr (KIND == kQ8_0) {
    w0 ^= 0x80808080u;  // signed byte q -> q + 128
    w1 ^= 0x80808080u;
    off = 8388736.0f;   // 2^23 + 128
  } else {
    const int sh = (part >> 1) * 4;  // parts 0,1: low nibbles; 2,3: high nibbles
    w0 = (w0 >> sh) & 0x0F0F0F0Fu;
    w1 = (w1 >> sh) & 0x0F0F0F0Fu;
    off = 8388616.0f;   // 2^23 + 8
  }
  const uint64_t o2 = pack2(-off, -off), d2 = pack2(d, d);
#pragma unroll
  for (int k = 0; k < 4; k += 2) {
    // x - off as fma(x, 1, -off): one rounding, exact here
    const uint64_t a = fma2(pack2(byte_as_float(w0, k), byte_as_float(w0, k + 1)),
                            pack2(1.0f, 1.0f), o2);
    const uint64_t b = fma2(pack2(byte_as_float(w1, k), byte_as_float(w1, k + 1)),
                            pack2(1.0f, 1.0f), o2);
    unpack2(mul2(a, d2), v[k], v[k + 1]);
    unpack2(mul2(b, d2), v[4 + k], v[4 + k + 1]);
  }
}

template <int OT>
__device__ __forceinline__ void store8(void* y, int64_t e0, const float (&v)[8], bool vec) {
  if (vec) {
    if constexpr (OT == kF32) {
      uint4* dst = reinterpret_cast<uint4*>(static_cast<float*>(y) + e0);
      dst[0] = make_uint4(__float_as_uint(v[0]), __float_as_uint(v[1]), __float_as_uint(v[2]),
                          __float_as_uint(v[3]));
      dst[1] = make_uint4(__float_as_uint(v[4]), __float_as_uint(v[5]), __float_as_uint(v[6]),
                          __float_as_uint(v[7]));
    } else {
      *reinterpret_cast<uint4*>(static_cast<uint16_t*>(y) + e0) =
          make_uint4(narrow2<OT>(v[0], v[1]), narrow2<OT>(v[2], v[3]), narrow2<OT>(v[4], v[5]),
                     narrow2<OT>(v[6], v[7]));
    }
  } else {
#pragma unroll
    for (int k = 0; k < 8; ++k) store_elem<OT>(y, e0 + k, v[k]);
  }
}

template <int KIND, int OT>
__global__ void __launch_bounds__(kGThreads) gguf_kernel(const GParams p) {
  constexpr int BB = GTraits<KIND>::BB;
  constexpr int STEP_BLOCKS = kGGroup * kGUnroll;  // 32
  constexpr int STEP_BYTES = STEP_BLOCKS * BB;     // 1088 or 576, multiples of 16
  constexpr int STEP_CHUNKS = STEP_BYTES / 16;     // 68 or 36
  constexpr int LOADS = (STEP_CHUNKS + 31) / 32;   // per lane: 3 or 2
  // 16 bytes of padding: the 8-byte reads of the last block load one aligned
  // word past the block
  __shared__ __align__(16) uint8_t buf[kGThreads / 32][STEP_BYTES + 16];

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  uint8_t* wb = buf[warp];
  const int64_t nsteps = (p.n_blocks + STEP_BLOCKS - 1) / STEP_BLOCKS;
  const int64_t nwarps = static_cast<int64_t>(gridDim.x) * (kGThreads / 32);
  pdl_release();
  pdl_wait();  // blocks and y may belong to the previous kernel

  // 16-byte chunks of a whole step, prefetched into registers one step ahead
  auto full_step = [&](int64_t g) {
    return p.vec && g < nsteps && (g + 1) * STEP_BLOCKS <= p.n_blocks;
  };
  auto fetch = [&](int64_t g, uint4 (&v)[LOADS]) {
    const uint4* src = reinterpret_cast<const uint4*>(p.blocks + g * STEP_BLOCKS * BB);
#pragma unroll
    for (int i = 0; i < LOADS; ++i) {
      const int c = lane + 32 * i;
      if (c < STEP_CHUNKS) v[i] = __ldg(src + c);
    }
  };
  uint4 vn[LOADS];
  int64_t g = static_cast<int64_t>(blockIdx.x) * (kGThreads / 32) + warp;
  if (full_step(g)) fetch(g, vn);

  for (; g < nsteps; g += nwarps) {
    const int64_t blk0 = g * STEP_BLOCKS;
    const int nblk = static_cast<int>(min(static_cast<int64_t>(STEP_BLOCKS), p.n_blocks - blk0));
    if (full_step(g)) {
#pragma unroll
      for (int i = 0; i < LOADS; ++i) {
        const int c = lane + 32 * i;
        if (c < STEP_CHUNKS) reinterpret_cast<uint4*>(wb)[c] = vn[i];
      }
      if (full_step(g + nwarps)) fetch(g + nwarps, vn);
    } else {
      const uint8_t* src = p.blocks + blk0 * BB;
      for (int i = lane; i < nblk * BB; i += 32) wb[i] = src[i];
    }
    __syncwarp();

    const int part = lane & 3;
#pragma unroll
    for (int u = 0; u < kGUnroll; ++u) {
      const int bl = u * kGGroup + (lane >> 2);
      if (bl < nblk) {
        float v[8];
        gguf_decode8<KIND, OT>(wb + bl * BB, part, v);
        store8<OT>(p.y, (blk0 + bl) * 32 + part * 8, v, p.vec != 0);
      }
    }
    __syncwarp();
  }
}

}  // namespace bq
