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
// Kernel design.  A warp takes groups of 8 blocks (272 B for Q8_0, 144 B for
// Q4_0: both whole multiples of 16 bytes, so a group of an aligned stream
// starts 16-byte aligned).  The group is staged into the warp's shared buffer
// with 16-byte loads, then lane l decodes 8 outputs of block l/4 and writes
// them as one 16-byte store, so each warp store covers 512 contiguous bytes of
// bf16 output.  Bytes become floats with the 2^23 trick: a byte b placed in
// the low mantissa bits of 2^23 is the float 2^23 + b, and subtracting
// 2^23 + offset is exact.  Unaligned streams and the last partial group are
// staged byte by byte.
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
constexpr int kGGroup = 8;  // blocks per warp step

template <int KIND> struct GTraits;
template <> struct GTraits<kQ8_0> { static constexpr int BB = 34; };
template <> struct GTraits<kQ4_0> { static constexpr int BB = 18; };

// byte k of w placed in the low mantissa of 2^23: the float 2^23 + byte
__device__ __forceinline__ float byte_as_float(uint32_t w, int k) {
  return __uint_as_float(__byte_perm(w, 0x4B000000u, 0x7540u + k));
}

template <int KIND, int OT>
__global__ void __launch_bounds__(kGThreads) gguf_kernel(const GParams p) {
  constexpr int BB = GTraits<KIND>::BB;
  constexpr int GBYTES = kGGroup * BB;  // 272 or 144, multiples of 16
  __shared__ __align__(16) uint8_t buf[kGThreads / 32][GBYTES];

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  uint8_t* wb = buf[warp];
  const int64_t ngroups = (p.n_blocks + kGGroup - 1) / kGGroup;
  const int64_t nwarps = static_cast<int64_t>(gridDim.x) * (kGThreads / 32);

  for (int64_t g = static_cast<int64_t>(blockIdx.x) * (kGThreads / 32) + warp; g < ngroups;
       g += nwarps) {
    const int64_t blk0 = g * kGGroup;
    const int nblk = static_cast<int>(min(static_cast<int64_t>(kGGroup), p.n_blocks - blk0));
    const uint8_t* src = p.blocks + blk0 * BB;
    if (p.vec && nblk == kGGroup) {
      if (lane < GBYTES / 16)
        reinterpret_cast<uint4*>(wb)[lane] = __ldg(reinterpret_cast<const uint4*>(src) + lane);
    } else {
      for (int i = lane; i < nblk * BB; i += 32) wb[i] = src[i];
    }
    __syncwarp();

    const int bl = lane >> 2, part = lane & 3;
    if (bl < nblk) {
      const uint8_t* bp = wb + bl * BB;
      const float d = __half2float(*reinterpret_cast<const __half*>(bp));
      // 8 quant bytes (2-byte aligned in the buffer)
      const uint8_t* qp = bp + 2 + (KIND == kQ8_0 ? 8 * part : 8 * (part & 1));
      const unsigned short* q16 = reinterpret_cast<const unsigned short*>(qp);
      uint32_t w0 = static_cast<uint32_t>(q16[0]) | (static_cast<uint32_t>(q16[1]) << 16);
      uint32_t w1 = static_cast<uint32_t>(q16[2]) | (static_cast<uint32_t>(q16[3]) << 16);
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
      float v[8];
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        v[k] = __fmul_rn(__fsub_rn(byte_as_float(w0, k), off), d);
        v[4 + k] = __fmul_rn(__fsub_rn(byte_as_float(w1, k), off), d);
      }
      const int64_t e0 = (blk0 + bl) * 32 + part * 8;
      if (p.vec) {
        if constexpr (OT == kF32) {
          uint4* dst = reinterpret_cast<uint4*>(static_cast<float*>(p.y) + e0);
          dst[0] = make_uint4(__float_as_uint(v[0]), __float_as_uint(v[1]), __float_as_uint(v[2]),
                              __float_as_uint(v[3]));
          dst[1] = make_uint4(__float_as_uint(v[4]), __float_as_uint(v[5]), __float_as_uint(v[6]),
                              __float_as_uint(v[7]));
        } else {
          uint4* dst = reinterpret_cast<uint4*>(static_cast<uint16_t*>(p.y) + e0);
          *dst = make_uint4(narrow2<OT>(v[0], v[1]), narrow2<OT>(v[2], v[3]),
                            narrow2<OT>(v[4], v[5]), narrow2<OT>(v[6], v[7]));
        }
      } else {
#pragma unroll
        for (int k = 0; k < 8; ++k) store_elem<OT>(p.y, e0 + k, v[k]);
      }
    }
    __syncwarp();
  }
}

}  // namespace bq
