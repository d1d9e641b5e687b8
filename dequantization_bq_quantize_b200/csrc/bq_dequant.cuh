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
// needs one absmax.  Each thread handles four chunks a grid-stride apart per
// iteration with all loads issued first.  Buffers that are not aligned for the
// vector path, and the elements after the last whole chunk, are done one
// element per thread.
#pragma once

#include "bq_common.cuh"

namespace bq {

struct DParams {
  const uint8_t* q;
  const float* absmax;
  const float* code;
  void* y;
  int64_t n;
  int64_t nchunks;   // whole 16-byte output chunks taken by the vector path
  int32_t bs_log2;
  int32_t vec;
};

constexpr int kDThreads = 256;

template <int E, int OT>
struct DTraits {
  static constexpr int OB = OT == kF32 ? 4 : 2;       // output element bytes
  static constexpr int CE = 16 / OB;                  // elements per chunk
  static constexpr int QB = E == 16 ? CE / 2 : CE;    // code bytes per chunk
};

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

// Code index of element e (0..CE-1) of a chunk whose code bytes are in c.
template <int E>
__device__ __forceinline__ uint32_t chunk_code(uint2 c, int e) {
  if constexpr (E == 16) {
    const uint32_t byte = (c.x >> ((e >> 1) << 3)) & 0xffu;
    return (e & 1) ? (byte & 15u) : (byte >> 4);
  } else {
    const uint32_t word = e < 4 ? c.x : c.y;
    return (word >> ((e & 3) << 3)) & 0xffu;
  }
}

template <int E, int OT>
__device__ __forceinline__ uint4 decode_chunk(uint2 c, float A, const float* sc) {
  constexpr int CE = DTraits<E, OT>::CE;
  float v[CE];
#pragma unroll
  for (int e = 0; e < CE; ++e) v[e] = __fmul_rn(sc[chunk_code<E>(c, e)], A);
  if constexpr (OT == kF32) {
    return make_uint4(__float_as_uint(v[0]), __float_as_uint(v[1]), __float_as_uint(v[2]),
                      __float_as_uint(v[3]));
  } else {
    return make_uint4(narrow2<OT>(v[0], v[1]), narrow2<OT>(v[2], v[3]), narrow2<OT>(v[4], v[5]),
                      narrow2<OT>(v[6], v[7]));
  }
}

template <int E, int OT>
__global__ void __launch_bounds__(kDThreads) dequant_kernel(const DParams p) {
  __shared__ float sc[E];
  for (int i = threadIdx.x; i < E; i += blockDim.x) sc[i] = p.code[i];
  __syncthreads();

  using T = DTraits<E, OT>;
  const int64_t gtid = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  const int64_t gsz = static_cast<int64_t>(gridDim.x) * blockDim.x;

  if (p.vec) {
    constexpr int U = 4;
    uint4* y4 = static_cast<uint4*>(p.y);
    for (int64_t base = gtid; base < p.nchunks; base += U * gsz) {
      uint2 c[U];
      float A[U];
#pragma unroll
      for (int u = 0; u < U; ++u) {
        const int64_t ch = base + u * gsz;
        if (ch < p.nchunks) {
          c[u] = load_codes<T::QB>(p.q, ch);
          A[u] = __ldg(p.absmax + ((ch * T::CE) >> p.bs_log2));
        }
      }
#pragma unroll
      for (int u = 0; u < U; ++u) {
        const int64_t ch = base + u * gsz;
        if (ch < p.nchunks) y4[ch] = decode_chunk<E, OT>(c[u], A[u], sc);
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
    store_elem<OT>(p.y, i, __fmul_rn(sc[idx], p.absmax[i >> p.bs_log2]));
  }
}

}  // namespace bq
