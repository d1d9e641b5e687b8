// bq_dequant.cuh - blockwise dequantization (sm_100a).
//
// y_i = narrow(RN(code[idx_i] * absmax[i / blocksize])), the inverse map of the
// blockwise quantization of "bitsandbytes PR #2052": a streaming gather from
// the codebook (held in shared memory) fused with the scale multiply and the
// bf16 / fp16 cast.
//
// Kernel design.  The output is cut into 16-byte chunks (8 elements of a
// 16-bit type, 4 of fp32); one thread makes one chunk, so every warp-wide
// store is 512 contiguous bytes and every warp-wide code load is contiguous
// too.  A chunk never straddles a quantization block (blocksize >= 32), so it
// needs one absmax.  Each thread handles eight chunks 32 apart per iteration
// (its warp's eight 512-byte stores are contiguous), with all loads issued
// first.  (Issuing the next iteration's loads
// before decoding these was tried and measured slower: the extra registers
// cost more occupancy than the overlap won.)
// 4-bit codes: a byte holds the codes of two neighbouring elements, so the
// shared table is indexed by the whole byte and holds the pair
// (code[byte >> 4], code[byte & 15]): one 64-bit shared load and one packed
// fp32x2 multiply per two elements.  8-bit codes: one 32-bit load per element,
// multiplied in pairs.  Buffers that are not aligned for the vector path, and
// the elements after the last whole chunk, are done one element per thread.
//
// Compressed statistics ("bitsandbytes PR #2052", Summary: the absmax array of
// NF4 storage is itself quantized blockwise with the General8 map): with
// NESTED, block b's scale is rebuilt in the kernel as
// A_b = RN(code2[qa[b]] * absmax2[b / blocksize2]) - the value the
// statistics' own dequantization would have stored - from a 256-entry shared
// table, so no fp32 absmax array is written or read.
#pragma once

#include "bq_search.cuh"

namespace bq {

struct DParams {
  const uint8_t* q;
  const float* absmax;   // plain statistics
  const float* code;
  void* y;
  int64_t n;
  int64_t nchunks;   // whole 16-byte output chunks taken by the vector path
  int32_t bs_log2;
  int32_t vec;
  // compressed statistics (NESTED kernels only)
  const uint8_t* qa;       // one code of code2 per block
  const float* absmax2;    // one scale per blocksize2 blocks
  const float* code2;      // 256 entries
  int32_t bs2_log2;
};

constexpr int kDThreads = 256;
constexpr int kDUnroll = 8;

template <int E, int OT>
struct DTraits {
  static constexpr int OB = OT == kF32 ? 4 : 2;       // output element bytes
  static constexpr int CE = 16 / OB;                  // elements per chunk
  static constexpr int QB = E == 16 ? CE / 2 : CE;    // code bytes per chunk
};

template <int E, bool NESTED>
struct DSmem {
  // E == 16: pair[b] = (code[b >> 4], code[b & 15]); E == 256: code[b]
  float t[E == 16 ? 512 : 256];
  float code[E];
  float code2[NESTED ? 256 : 1];
};

// Scale of quantization block b: stored, or rebuilt from its code and the
// second-level scale.
template <bool NESTED, int E>
__device__ __forceinline__ float block_scale(const DParams& p, const DSmem<E, NESTED>& s,
                                             int64_t b) {
  if constexpr (NESTED) {
    return __fmul_rn(s.code2[__ldg(p.qa + b)], __ldg(p.absmax2 + (b >> p.bs2_log2)));
  } else {
    return __ldg(p.absmax + b);
  }
}

template <int QB>
__device__ __forceinline__ uint2 load_codes(const uint8_t* __restrict__ q, int64_t chunk) {
  if constexpr (QB == 8) {
    return __ldg(reinterpret_cast<const uint2*>(q) + chunk);
  } else if constexpr (QB == 4) {
    return make_uint2(__ldg(reinterpret_cast<const uint32_t*>(q) + chunk), 0u);
  } else {
    return make_uint2(__ldg(reinterpret_cast<const unsigned short*>(q) + chunk), 0u);
  }
}

// Two outputs from one code byte pair index / two code bytes, times A.  The
// table reads are asm with no memory dependence: their addresses come from
// code bytes loaded from global memory after the table was built and
// __syncthreads, and that data dependence keeps them after the build.
// STRIDE: bytes between consecutive table entries (8 / 4 for a plain table;
// 128 for a table replicated per lane, t_base then pointing at this lane's
// copy).
template <int E, int STRIDE = (E == 16 ? 8 : 4)>
__device__ __forceinline__ void decode_pair(uint2 c, int k, uint32_t t_base, uint64_t a2,
                                            float& v0, float& v1) {
  if constexpr (E == 16) {
    // byte k of the chunk's code word: elements 2k (high nibble), 2k+1 (low)
    const uint32_t byte = __byte_perm(c.x, 0u, 0x4440u + k);
    uint2 pr;
    asm("ld.shared.v2.u32 {%0, %1}, [%2];" : "=r"(pr.x), "=r"(pr.y) : "r"(t_base + byte * STRIDE));
    unpack2(mul2(pack2(__uint_as_float(pr.x), __uint_as_float(pr.y)), a2), v0, v1);
  } else {
    const uint32_t word = k < 2 ? c.x : c.y;
    const uint32_t b0 = __byte_perm(word, 0u, 0x4440u + 2 * (k & 1));
    const uint32_t b1 = __byte_perm(word, 0u, 0x4441u + 2 * (k & 1));
    float c0, c1;
    asm("ld.shared.f32 %0, [%1];" : "=f"(c0) : "r"(t_base + b0 * STRIDE));
    asm("ld.shared.f32 %0, [%1];" : "=f"(c1) : "r"(t_base + b1 * STRIDE));
    unpack2(mul2(pack2(c0, c1), a2), v0, v1);
  }
}

template <int E, int OT, int STRIDE = (E == 16 ? 8 : 4)>
__device__ __forceinline__ uint4 decode_chunk(uint2 c, float A, uint32_t t_base) {
  constexpr int CE = DTraits<E, OT>::CE;
  const uint64_t a2 = pack2(A, A);
  float v[CE];
#pragma unroll
  for (int k = 0; k < CE / 2; ++k)
    decode_pair<E, STRIDE>(c, k, t_base, a2, v[2 * k], v[2 * k + 1]);
  if constexpr (OT == kF32) {
    return make_uint4(__float_as_uint(v[0]), __float_as_uint(v[1]), __float_as_uint(v[2]),
                      __float_as_uint(v[3]));
  } else {
    return make_uint4(narrow2<OT>(v[0], v[1]), narrow2<OT>(v[2], v[3]), narrow2<OT>(v[4], v[5]),
                      narrow2<OT>(v[6], v[7]));
  }
}

template <int E, int OT, bool NESTED>
__global__ void __launch_bounds__(kDThreads) dequant_kernel(const DParams p) {
  __shared__ DSmem<E, NESTED> s;
  pdl_release();
  pdl_wait();  // codes, absmax, codebook and y may belong to the previous kernel
  for (int i = threadIdx.x; i < E; i += blockDim.x) s.code[i] = p.code[i];
  if constexpr (NESTED)
    for (int i = threadIdx.x; i < 256; i += blockDim.x) s.code2[i] = p.code2[i];
  __syncthreads();
  if constexpr (E == 16) {
    for (int b = threadIdx.x; b < 256; b += blockDim.x) {
      s.t[2 * b] = s.code[b >> 4];
      s.t[2 * b + 1] = s.code[b & 15];
    }
  } else {
    for (int b = threadIdx.x; b < 256; b += blockDim.x) s.t[b] = s.code[b];
  }
  __syncthreads();
  const uint32_t t_base = smem_u32(s.t);

  using T = DTraits<E, OT>;
  const int64_t gtid = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  const int64_t gsz = static_cast<int64_t>(gridDim.x) * blockDim.x;

  if (p.vec) {
    constexpr int U = kDUnroll;
    uint4* y4 = static_cast<uint4*>(p.y);
    // a warp writes U * 512 contiguous bytes per iteration (chunks base,
    // base + 32, ... for its lanes), the warps of a CTA side by side: longer
    // runs of output per DRAM row than a grid-stride between a thread's
    // chunks (266 -> 254 us for NF4 at n = 2^29 bf16)
    const int64_t lane_ = threadIdx.x & 31;
    const int64_t wstride = (gsz >> 5) * U * 32;
    for (int64_t base = (gtid >> 5) * U * 32 + lane_; base < p.nchunks; base += wstride) {
      uint2 c[U];
      float A[U];
      uint32_t qa[U];  // NESTED: the block's statistics code, looked up after the loads
#pragma unroll
      for (int u = 0; u < U; ++u) {
        const int64_t ch = base + u * 32;
        if (ch < p.nchunks) {
          c[u] = load_codes<T::QB>(p.q, ch);
          const int64_t b = (ch * T::CE) >> p.bs_log2;
          if constexpr (NESTED) {
            qa[u] = __ldg(p.qa + b);
            A[u] = __ldg(p.absmax2 + (b >> p.bs2_log2));
          } else {
            A[u] = __ldg(p.absmax + b);
          }
        }
      }
#pragma unroll
      for (int u = 0; u < U; ++u) {
        const int64_t ch = base + u * 32;
        if (ch < p.nchunks) {
          if constexpr (NESTED) A[u] = __fmul_rn(s.code2[qa[u]], A[u]);
          y4[ch] = decode_chunk<E, OT>(c[u], A[u], t_base);
        }
      }
    }
  }
  // element-wise: everything (no vector path) or the tail after the chunks
  const int64_t first = p.vec ? p.nchunks * T::CE : 0;
  for (int64_t i = first + gtid; i < p.n; i += gsz) {
    uint32_t idx;
    if constexpr (E == 16) {
      const uint32_t byte = p.q[i >> 1];
      idx = (i & 1) ? (byte & 15u) : (byte >> 4);
    } else {
      idx = p.q[i];
    }
    store_elem<OT>(p.y, i, __fmul_rn(s.code[idx], block_scale<NESTED>(p, s, i >> p.bs_log2)));
  }
}

}  // namespace bq
