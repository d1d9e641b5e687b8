// bq_gguf.cuh - GGUF block dequantization (sm_100a): Q8_0, Q4_0, Q4_1, Q5_0,
// Q5_1, Q2_K, Q3_K, Q4_K, Q5_K, Q6_K, and the BF16 conversion.
//
// Formats.  Q8_0 and Q4_0 as on "ComfyUI-GGUF PR #472, Cache device-side
// constants in dequant kernels", Problem section and Verification table:
//   Q8_0 block = fp16 d + 32 signed bytes q:       y = d * q
//   Q4_0 block = fp16 d + 16 bytes qs, shifts [0, 4]: y[j] = d * ((qs[j] & 15) - 8),
//                                                    y[16 + j] = d * ((qs[j] >> 4) - 8)
// The other rows of that table follow the GGUF block layouts (the page names
// the types without spelling them out):
//   Q4_1 = fp16 d, fp16 m, qs[16]:            y = d * nibble + m
//   Q5_0 = fp16 d, u32 qh, qs[16]:            y = d * (q - 16), q = nibble | bit e of qh << 4
//   Q5_1 = fp16 d, fp16 m, u32 qh, qs[16]:    y = d * q + m
//   Q4_K = super-block of 256: fp16 d, fp16 dmin, 12 bytes of packed 6-bit
//          scales and mins for 8 sub-blocks of 32, qs[128]:  y = d*sc*q - dmin*mn
//   Q6_K = super-block of 256: ql[128], qh[64], int8 scales[16], fp16 d:
//          y = d * sc * (q - 32), q = 4 bits of ql | 2 bits of qh << 4
//   Q2_K = super-block of 256: scales[16] (min << 4 | scale), qs[64], fp16 d,
//          fp16 dmin: y = d*sc*q - dmin*mn, q 2 bits
//   Q3_K = super-block of 256: hmask[32], qs[64], 12 bytes of packed 6-bit
//          scales, fp16 d: y = d*(s - 32)*q, q = 2 bits - (hmask bit ? 0 : 4)
//   Q5_K = super-block of 256: fp16 d, fp16 dmin, scales as Q4_K, qh[32],
//          qs[128]: y = d*sc*q - dmin*mn, q = nibble | qh bit << 4
// Every product here is exact in fp32 (an 11-bit d times at most 7 + 5 more
// bits), so the only rounding before the narrowing is the add of a min,
// done as one fma: the narrowed output is the correctly rounded value.  The
// page's point - no per-call host-to-device constants - holds trivially here:
// shifts and offsets live in registers.
//
// Kernel design.  A lane always decodes 8 consecutive outputs of one block
// and writes them as one 16-byte store (bf16), so a warp pass writes 512
// contiguous bytes: 8 blocks of 32 (lanes 4b..4b+3 share block b) or one
// super-block of 256.  A warp step covers 32 blocks (8 super-blocks), a whole
// number of 16-byte chunks in every format, so in a 16-byte aligned stream
// every step starts aligned; the warp stages a step into its shared buffer
// with up to four 16-byte loads per lane, fetched into registers one step
// ahead.  Bytes become floats with the 2^23 trick: a byte b placed in the low
// mantissa bits of 2^23 is the float 2^23 + b, and subtracting 2^23 + offset
// is exact.  Unaligned streams and the last partial step are staged byte by
// byte.
#pragma once

#include <type_traits>

#include "bq_common.cuh"

namespace bq {

enum : int {
  kQ8_0 = 0, kQ4_0 = 1, kQ4_1 = 2, kQ5_0 = 3, kQ5_1 = 4, kQ4_K = 5, kQ6_K = 6,
  kQ2_K = 7, kQ3_K = 8, kQ5_K = 9
};

struct GParams {
  const uint8_t* blocks;
  void* y;
  int64_t n_blocks;
  int32_t vec;   // blocks and y are 16-byte aligned
};

constexpr int kGThreads = 256;

// BB: bytes per block; EPB: outputs per block; QS: offset of the nibble bytes;
// QH: offset of the 32 high bits (Q5); MIN: the block carries an fp16 min
template <int KIND> struct GTraits;
template <> struct GTraits<kQ8_0> { static constexpr int BB = 34, EPB = 32, QS = 2, QH = 0; static constexpr bool MIN = false; };
template <> struct GTraits<kQ4_0> { static constexpr int BB = 18, EPB = 32, QS = 2, QH = 0; static constexpr bool MIN = false; };
template <> struct GTraits<kQ4_1> { static constexpr int BB = 20, EPB = 32, QS = 4, QH = 0; static constexpr bool MIN = true; };
template <> struct GTraits<kQ5_0> { static constexpr int BB = 22, EPB = 32, QS = 6, QH = 2; static constexpr bool MIN = false; };
template <> struct GTraits<kQ5_1> { static constexpr int BB = 24, EPB = 32, QS = 8, QH = 4; static constexpr bool MIN = true; };
template <> struct GTraits<kQ4_K> { static constexpr int BB = 144, EPB = 256, QS = 16, QH = 0; static constexpr bool MIN = true; };
template <> struct GTraits<kQ6_K> { static constexpr int BB = 210, EPB = 256, QS = 0, QH = 128; static constexpr bool MIN = false; };
template <> struct GTraits<kQ2_K> { static constexpr int BB = 84, EPB = 256, QS = 16, QH = 0; static constexpr bool MIN = true; };
template <> struct GTraits<kQ3_K> { static constexpr int BB = 110, EPB = 256, QS = 32, QH = 0; static constexpr bool MIN = false; };
template <> struct GTraits<kQ5_K> { static constexpr int BB = 176, EPB = 256, QS = 48, QH = 16; static constexpr bool MIN = true; };

// blocks per warp step: 32 blocks of 32 or 8 super-blocks of 256
template <int KIND> struct GStep { static constexpr int value = GTraits<KIND>::EPB == 32 ? 32 : 8; };

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

// Eight bytes at a shared address whose remainder mod 8 is BA, known at
// compile time (BA = -1: unknown, any 2-byte aligned address).  K-quant
// super-blocks sit at u * BB bytes of an 8-byte aligned staging buffer and
// are read at multiples of 8 inside the block, so pass u of a warp step reads
// at remainder (u * BB) mod 8: one 64-bit load, two 32-bit loads, or three and
// a fixed 16-bit funnel shift (Q3_K's 110- and Q6_K's 210-byte blocks
// alternate).
template <int BA>
__device__ __forceinline__ void load8(const uint8_t* ptr, uint32_t& w0, uint32_t& w1) {
  if constexpr (BA < 0) {
    load8_at2(ptr, w0, w1);
  } else if constexpr (BA == 0) {
    const uint2 q = *reinterpret_cast<const uint2*>(ptr);
    w0 = q.x;
    w1 = q.y;
  } else if constexpr (BA == 4) {
    const uint32_t* wp = reinterpret_cast<const uint32_t*>(ptr);
    w0 = wp[0];
    w1 = wp[1];
  } else {
    static_assert(BA == 2 || BA == 6, "2-byte aligned reads only");
    const uint32_t* wp = reinterpret_cast<const uint32_t*>(ptr - 2);
    const uint32_t x0 = wp[0], x1 = wp[1], x2 = wp[2];
    w0 = __funnelshift_r(x0, x1, 16);
    w1 = __funnelshift_r(x1, x2, 16);
  }
}

__device__ __forceinline__ float half_at(const uint8_t* p) {
  return __half2float(*reinterpret_cast<const __half*>(p));
}

// bit k (k < 4) of a nibble moved to bit 4 of byte k: the four shifted copies
// x, x << 7, x << 14, x << 21 do not overlap, so the product is their OR
__device__ __forceinline__ uint32_t spread4_to_bit4(uint32_t x4) {
  return ((x4 * 0x00204081u) & 0x01010101u) << 4;
}

// v[k] = (float(2^23 + byte k) - (2^23 + off)) * s, or with a min:
// fma(float(2^23 + byte k) - 2^23, s, m); two lanes per packed op
template <bool MIN>
__device__ __forceinline__ void bytes_to_values(uint32_t w0, uint32_t w1, float off, float s,
                                                float m, float (&v)[8]) {
  const uint64_t o2 = pack2(-off, -off), s2 = pack2(s, s), one2 = pack2(1.0f, 1.0f);
  const uint64_t m2 = pack2(m, m);
#pragma unroll
  for (int k = 0; k < 4; k += 2) {
    // x - off as fma(x, 1, -off): one rounding, exact here
    const uint64_t a = fma2(pack2(byte_as_float(w0, k), byte_as_float(w0, k + 1)), one2, o2);
    const uint64_t b = fma2(pack2(byte_as_float(w1, k), byte_as_float(w1, k + 1)), one2, o2);
    if constexpr (MIN) {
      unpack2(fma2(a, s2, m2), v[k], v[k + 1]);
      unpack2(fma2(b, s2, m2), v[4 + k], v[4 + k + 1]);
    } else {
      unpack2(mul2(a, s2), v[k], v[k + 1]);
      unpack2(mul2(b, s2), v[4 + k], v[4 + k + 1]);
    }
  }
}

// Decode outputs 8*part .. 8*part+7 of the block at bp (part < EPB / 8).
// BA: bp's remainder mod 8 when known at compile time, else -1.
template <int KIND, int BA = -1>
__device__ __forceinline__ void gguf_decode8(const uint8_t* bp, int part, float (&v)[8]) {
  using T = GTraits<KIND>;
  uint32_t w0, w1;
  if constexpr (KIND == kQ8_0) {
    load8_at2(bp + 2 + 8 * part, w0, w1);
    w0 ^= 0x80808080u;  // signed byte q -> q + 128
    w1 ^= 0x80808080u;
    bytes_to_values<false>(w0, w1, 8388736.0f /* 2^23 + 128 */, half_at(bp), 0.0f, v);
  } else if constexpr (T::EPB == 32) {
    // nibble formats: parts 0, 1 are the low nibbles of qs[0..7], qs[8..15];
    // parts 2, 3 the high nibbles
    load8_at2(bp + T::QS + 8 * (part & 1), w0, w1);
    const int sh = (part >> 1) * 4;
    w0 = (w0 >> sh) & 0x0F0F0F0Fu;
    w1 = (w1 >> sh) & 0x0F0F0F0Fu;
    if constexpr (T::QH != 0) {
      const uint32_t hb = bp[T::QH + part];  // bits 8*part .. 8*part+7 of qh
      w0 |= spread4_to_bit4(hb & 15u);
      w1 |= spread4_to_bit4(hb >> 4);
    }
    const float d = half_at(bp);
    if constexpr (T::MIN) {
      bytes_to_values<true>(w0, w1, 8388608.0f /* 2^23 */, d, half_at(bp + 2), v);
    } else {
      const float off = KIND == kQ4_0 ? 8388616.0f /* 2^23 + 8 */ : 8388624.0f /* 2^23 + 16 */;
      bytes_to_values<false>(w0, w1, off, d, 0.0f, v);
    }
  } else if constexpr (KIND == kQ4_K) {
    // part = 8g + 4h + r: group g of 64 reads qs[32g + 8r ..], nibble half h,
    // sub-block 2g + h
    const int g = part >> 3, h = (part >> 2) & 1, r = part & 3;
    const int is = 2 * g + h, j = is & 3;
    const uint32_t A = bp[4 + j], B = bp[8 + j], C = bp[12 + j];
    const bool hi = is >= 4;
    const uint32_t sc = hi ? ((C & 15u) | ((A >> 6) << 4)) : (A & 63u);
    const uint32_t mn = hi ? ((C >> 4) | ((B >> 6) << 4)) : (B & 63u);
    const float a = half_at(bp) * static_cast<float>(sc);        // exact
    const float b = half_at(bp + 2) * static_cast<float>(mn);    // exact
    const uint2 q = *reinterpret_cast<const uint2*>(bp + 16 + 32 * g + 8 * r);  // 8-byte aligned
    w0 = (q.x >> (4 * h)) & 0x0F0F0F0Fu;
    w1 = (q.y >> (4 * h)) & 0x0F0F0F0Fu;
    bytes_to_values<true>(w0, w1, 8388608.0f, a, -b, v);
  } else if constexpr (KIND == kQ5_K) {
    // as Q4_K, plus bit 2g + h of qh[8r ..] as bit 4
    const int g = part >> 3, h = (part >> 2) & 1, r = part & 3;
    const int is = 2 * g + h, j = is & 3;
    const uint32_t A = bp[4 + j], B = bp[8 + j], C = bp[12 + j];
    const bool hi = is >= 4;
    const uint32_t sc = hi ? ((C & 15u) | ((A >> 6) << 4)) : (A & 63u);
    const uint32_t mn = hi ? ((C >> 4) | ((B >> 6) << 4)) : (B & 63u);
    const float a = half_at(bp) * static_cast<float>(sc);        // exact
    const float b = half_at(bp + 2) * static_cast<float>(mn);    // exact
    const uint2 q = *reinterpret_cast<const uint2*>(bp + 48 + 32 * g + 8 * r);  // 8-byte aligned
    const uint2 hb = *reinterpret_cast<const uint2*>(bp + 16 + 8 * r);
    w0 = ((q.x >> (4 * h)) & 0x0F0F0F0Fu) | (((hb.x >> is) & 0x01010101u) << 4);
    w1 = ((q.y >> (4 * h)) & 0x0F0F0F0Fu) | (((hb.y >> is) & 0x01010101u) << 4);
    bytes_to_values<true>(w0, w1, 8388608.0f, a, -b, v);
  } else if constexpr (KIND == kQ2_K) {
    // part = 16n + 4c + 2h + s: outputs 128n + 32c + 16h + 8s .., 2-bit field c
    // of qs[32n + 16h + 8s ..], sub-block part / 2
    const int n = part >> 4, c = (part >> 2) & 3, hh = (part >> 1) & 1, s8 = (part & 1) * 8;
    const uint32_t scb = bp[part >> 1];
    const float a = half_at(bp + 80) * static_cast<float>(scb & 15u);  // exact
    const float b = half_at(bp + 82) * static_cast<float>(scb >> 4);   // exact
    load8<BA>(bp + 16 + 32 * n + 16 * hh + s8, w0, w1);
    w0 = (w0 >> (2 * c)) & 0x03030303u;
    w1 = (w1 >> (2 * c)) & 0x03030303u;
    bytes_to_values<true>(w0, w1, 8388608.0f, a, -b, v);
  } else if constexpr (KIND == kQ3_K) {
    // part = 16n + 4c + 2h + s as Q2_K; bit 4n + c of hmask[16h + 8s ..]
    // clear means q - 4: the byte (low | hbit << 2) minus 4 is q
    const int n = part >> 4, c = (part >> 2) & 3, hh = (part >> 1) & 1, s8 = (part & 1) * 8;
    const int i = part >> 1;  // sub-block
    const uint32_t lo4 = i < 8 ? (bp[96 + i] & 15u) : (bp[96 + i - 8] >> 4);
    const uint32_t hi2 = (bp[104 + (i & 3)] >> (2 * (i >> 2))) & 3u;
    const int scale = static_cast<int>(lo4 | (hi2 << 4)) - 32;
    const float a = half_at(bp + 108) * static_cast<float>(scale);  // exact
    uint32_t m0, m1;
    load8<BA>(bp + 32 + 32 * n + 16 * hh + s8, w0, w1);
    load8<BA>(bp + 16 * hh + s8, m0, m1);
    const int hs = 4 * n + c;
    w0 = ((w0 >> (2 * c)) & 0x03030303u) | (((m0 >> hs) & 0x01010101u) << 2);
    w1 = ((w1 >> (2 * c)) & 0x03030303u) | (((m1 >> hs) & 0x01010101u) << 2);
    bytes_to_values<false>(w0, w1, 8388612.0f /* 2^23 + 4 */, a, 0.0f, v);
  } else {  // kQ6_K
    // part = 16n + 4c + r: half n, 32-element chunk c, outputs 8r..8r+7 of it
    const int n = part >> 4, c = (part >> 2) & 3, r = part & 3;
    uint32_t h0, h1;
    load8<BA>(bp + 64 * n + 32 * (c & 1) + 8 * r, w0, w1);
    load8<BA>(bp + 128 + 32 * n + 8 * r, h0, h1);
    const int sl = 4 * (c >> 1), sh = 2 * c;
    w0 = ((w0 >> sl) & 0x0F0F0F0Fu) | (((h0 >> sh) & 0x03030303u) << 4);
    w1 = ((w1 >> sl) & 0x0F0F0F0Fu) | (((h1 >> sh) & 0x03030303u) << 4);
    const int scale = static_cast<int8_t>(bp[192 + 8 * n + (r >> 1) + 2 * c]);
    const float a = half_at(bp + 208) * static_cast<float>(scale);  // exact
    bytes_to_values<false>(w0, w1, 8388640.0f /* 2^23 + 32 */, a, 0.0f, v);
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

// f(integral_constant<int, U>) for U = B .. E-1, in order
template <int B, int E, typename F>
__device__ __forceinline__ void static_for(F&& f) {
  if constexpr (B < E) {
    f(std::integral_constant<int, B>{});
    static_for<B + 1, E>(f);
  }
}

template <int KIND, int OT>
__global__ void __launch_bounds__(kGThreads) gguf_kernel(const GParams p) {
  using T = GTraits<KIND>;
  constexpr int BB = T::BB;
  constexpr int LPB = T::EPB / 8;                  // lanes per block: 4 or 32
  constexpr int GROUP = 32 / LPB;                  // blocks per warp pass: 8 or 1
  constexpr int STEP_BLOCKS = GStep<KIND>::value;
  constexpr int UNROLL = STEP_BLOCKS / GROUP;      // warp passes per step: 4 or 8
  constexpr int STEP_BYTES = STEP_BLOCKS * BB;     // a multiple of 16 in every format
  constexpr int STEP_CHUNKS = STEP_BYTES / 16;
  constexpr int LOADS = (STEP_CHUNKS + 31) / 32;   // per lane: 2 to 4
  static_assert(STEP_BYTES % 16 == 0, "a step must be whole 16-byte chunks");
  // 16 bytes of padding: the 8-byte reads of the last block may load one
  // aligned word past the block.  Every warp's buffer starts 16-byte aligned.
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

    const int part = lane % LPB;
    // one pass per u; with one block per pass (K-quants) its offset u * BB,
    // and so the alignment of its reads, is a compile-time constant
    static_for<0, UNROLL>([&](auto uc) {
      constexpr int u = decltype(uc)::value;
      const int bl = u * GROUP + lane / LPB;
      if (bl < nblk) {
        float v[8];
        gguf_decode8<KIND, GROUP == 1 ? (u * BB) % 8 : -1>(wb + bl * BB, part, v);
        store8<OT>(p.y, (blk0 + bl) * T::EPB + part * 8, v, p.vec != 0);
      }
    });
    __syncwarp();
  }
}

// GGUF BF16 ("ComfyUI-GGUF PR #472", Verification table, BF16 row): plain
// bfloat16 values, widened exactly and narrowed to the output type (a copy
// for a bf16 output).  One thread per 8 values (16 bytes in); the elements
// after the last whole group, and unaligned buffers, one per thread.
struct BParams {
  const uint16_t* x;
  void* y;
  int64_t n;
  int64_t ngroups;  // whole groups of 8 taken by the vector path
};

template <int OT>
__global__ void __launch_bounds__(kGThreads) bf16_kernel(const BParams p) {
  pdl_release();
  pdl_wait();
  const int64_t gtid = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  const int64_t gsz = static_cast<int64_t>(gridDim.x) * blockDim.x;
  for (int64_t gi = gtid; gi < p.ngroups; gi += gsz) {
    const uint4 w = __ldg(reinterpret_cast<const uint4*>(p.x) + gi);
    if constexpr (OT == kBF16) {
      reinterpret_cast<uint4*>(p.y)[gi] = w;
    } else {
      const uint32_t ws[4] = {w.x, w.y, w.z, w.w};
      float v[8];
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        v[2 * k] = __uint_as_float(ws[k] << 16);
        v[2 * k + 1] = __uint_as_float(ws[k] & 0xffff0000u);
      }
      store8<OT>(p.y, gi * 8, v, true);
    }
  }
  for (int64_t i = p.ngroups * 8 + gtid; i < p.n; i += gsz) {
    const uint32_t h = p.x[i];
    if constexpr (OT == kBF16) static_cast<uint16_t*>(p.y)[i] = static_cast<uint16_t>(h);
    else store_elem<OT>(p.y, i, __uint_as_float(h << 16));
  }
}

}  // namespace bq
