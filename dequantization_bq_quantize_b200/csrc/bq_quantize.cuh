// bq_quantize.cuh - blockwise absmax codebook quantization (sm_100a).
//
// Method: "bitsandbytes PR #2052" (General8 / FP4 / NF4 blockwise
// quantization, block sizes 32..4096, full blocks and tails, FP16 / BF16 /
// FP32 inputs).  Per block: absmax, xn = x / absmax (IEEE fp32), nearest code
// (lowest index on ties), codes packed two per byte high nibble first
// (16-entry tables) or one per byte (256-entry tables).
//
// Kernel design.  A persistent grid (2 CTAs per SM) of 288-thread CTAs (320
// with the statistics warp): one producer warp streams 16 KiB input tiles (128 rows of 128 B) into a 4-stage
// shared-memory ring with 2-D TMA loads (128-byte swizzle, no multicast), and
// 8 consumer warps process each tile.  Consumer thread t owns 64 contiguous
// bytes (row t/2, half t%2), read with four conflict-free 16-byte shared
// loads thanks to the swizzle.  A quantization block spans TPB =
// blocksize * elem_bytes / 64 consecutive threads: its absmax is a shuffle-xor
// tree over TPB lanes (one integer warp reduction when TPB = 32); blocks
// wider than a warp (TPB > 32) get theirs from a statistics warp that reads
// each tile as it lands (stats_main), so no consumer warp waits for another.
// The stage is released as soon as the values are in registers.
//
// Per element the fast path costs about ten instructions:
//  - 16-bit inputs: absmax from packed two-lane max of absolute values
//    (NaN-propagating, so a block holding a NaN or inf is recognised by its
//    absmax and takes the safe path);
//  - xn two elements per instruction with the sm_100 fp32x2 FMA / MUL: for
//    16-bit inputs one product with the trailing term of a two-term
//    reciprocal and one FMA with its leading term (div_fast2_2term), for fp32
//    inputs Markstein's correction from the rounded reciprocal (no
//    per-element range check: see div_fast);
//  - the code from a bucket table (bq_search.cuh): one packed bucket
//    computation per pair, one 64-bit shared load and one compare per
//    element (16-entry tables: each lane reads its own interleaved copy, so
//    the loads never conflict on banks); 256-entry tables whose codes step by
//    one: one 32-bit shared load and one add per element (kModeLutI);
//  - codes inserted into the output words with bit-field inserts.
// Blocks whose absmax is outside [2^-60, 2^60] (or not finite), and codebooks
// without a bucket table, take the safe path: IEEE division where Markstein's
// form is not valid, and a clamped lookup.  Bytes of the input that do not
// fill a whole tile, and every input that is not 16-byte aligned, are handled
// one block per warp from global memory with IEEE division.
#pragma once

#include "bq_search.cuh"

namespace bq {

constexpr int kQConsumerWarps = 8;
constexpr int kQConsumers = kQConsumerWarps * 32;  // 256
constexpr int kTileBytes = 16384;
constexpr int kTileRows = 128;                     // rows of 128 bytes
constexpr int kStages = 4;
constexpr int kThreadBytes = kTileBytes / kQConsumers;  // 64
constexpr int kThreadWords = kThreadBytes / 4;           // 16
static_assert(kThreadBytes == 64, "thread owns four 16-byte chunks");

// Blocks that span more than one warp of consumers (TPB > 32 threads) get
// their absmax from a statistics warp instead of a reduction across the
// consumer warps: the statistics warp reads each tile as it lands, writes the
// absmax of its blocks to shared memory and signals an mbarrier, so the
// consumer warps never wait for one another (a cross-warp reduction put a
// CTA-wide barrier on every tile: bf16 blocksize 4096 ran at 0.72-0.76 of the
// measured copy bandwidth against 0.89-0.99 for smaller blocks).
template <int TPB> constexpr bool kStatsWarp = TPB > 32;
// 16-bit inputs with 16-entry tables (two or four blocks per tile) split the
// statistics work over two warps, block b to warp b % 2: one statistics warp
// adds its ~170 instructions per tile to a single SM sub-partition, which
// then limits the issue-bound kernel (bf16 NF4 blocksize 4096, 1 GiB:
// 258.4 -> 252.4 us).  256-entry tables keep one (their consumers need 96
// registers; 352-thread CTAs at two per SM allow 88), and fp32 inputs,
// which leave issue slots to spare, keep one.
template <int DT, int E, int TPB>
constexpr int kNumStats = TPB > 32 ? ((DT != kF32 && E == 16) ? 2 : 1) : 0;
template <int DT, int E, int TPB>
constexpr int q_threads() { return kQConsumers + 32 + 32 * kNumStats<DT, E, TPB>; }
constexpr int kQMaxTileBlocks = 4;   // blocks per tile when TPB > 32 (TPB >= 64)

template <int E>
struct QSmem {
  uint8_t stage[kStages][kTileBytes];  // 1024-byte aligned (128B swizzle)
  uint64_t full[kStages];
  uint64_t empty[kStages];
  uint64_t stats[kStages];             // statistics warp: the stage's absmax is ready
  float tamax[kStages][kQMaxTileBlocks];
  TableSmem tab;
  Lut<E> lut;
};

template <int E>
constexpr size_t qsmem_bytes() { return sizeof(QSmem<E>) + 1024; }

struct QParams {
  const void* x;
  int64_t n;
  const float* code;
  float* absmax;
  uint8_t* out;
  int64_t full_tiles;  // tiles streamed by TMA; the rest goes block by block
  int64_t nb;          // number of quantization blocks
  int32_t bs;
};

// ------------------------------------------------------ small helpers -----

__device__ __forceinline__ uint32_t bfi(uint32_t field, uint32_t base, int pos, int len) {
  uint32_t d;
  asm("bfi.b32 %0, %1, %2, %3, %4;" : "=r"(d) : "r"(field), "r"(base), "r"(pos), "r"(len));
  return d;
}

// Table read by shared-window address.  The asm has no memory dependence, so
// it is only ever fed addresses computed from tile data loaded after the
// mbarrier wait (itself after the table build and its barrier): the data
// dependence keeps it after both.
__device__ __forceinline__ uint2 lds_u64(uint32_t addr) {
  uint2 v;
  asm("ld.shared.v2.u32 {%0, %1}, [%2];" : "=r"(v.x), "=r"(v.y) : "r"(addr));
  return v;
}
__device__ __forceinline__ uint32_t lds_u32(uint32_t addr) {
  uint32_t v;
  asm("ld.shared.u32 %0, [%1];" : "=r"(v) : "r"(addr));
  return v;
}

template <int DT>
__device__ __forceinline__ float tile_elem(const uint32_t (&w)[kThreadWords], int j) {
  if constexpr (DT == kF32) return __uint_as_float(w[j]);
  else return widen_pair_elem<DT>(w[j >> 1], j & 1);
}

// Output bit position of element j in the thread's code words.
template <int E>
__device__ __forceinline__ constexpr int code_pos(int j) {
  if constexpr (E == 16) return (((j & 7) >> 1) << 3) + ((j & 1) ? 0 : 4);
  else return (j & 3) << 3;
}

// Codes of one thread: EPT elements -> OUT_BYTES bytes in NW words.
template <int DT, int E>
struct QOut {
  static constexpr int EPT = kThreadBytes / ElemBytes<DT>::value;
  static constexpr int BYTES = E == 16 ? EPT / 2 : EPT;
  static constexpr int NW = BYTES / 4;
  static constexpr int L = E == 16 ? 4 : 8;        // bits per code
  static constexpr int PER_WORD = 32 / L;
};

// ------------------------------------------------------ fast encoding -----

// Shared address of the bucket's entry.  For 16-entry tables `b` is already
// fma(xn, 15, 1.5 * 2^23) and t_base = &lut.r[0][lane % 16] -
// 128 * (0x4B400000 - 15), so bits(b) * 128 + t_base addresses this lane's
// copy of the bucket (32-bit wrap-around arithmetic).  For 256-entry tables b
// is xn and t_base = &lut.e[1537].
template <int E>
__device__ __forceinline__ uint32_t lut_addr(float b, uint32_t t_base) {
  if constexpr (E == 16) {
    return __float_as_uint(b) * 128u + t_base;
  } else {
    const uint32_t u = __float_as_uint(b);
    const uint32_t a = u & 0x7fffffffu;
    const uint32_t idx = (max(a, 0x33800000u) - 0x33800000u) >> 17;
    const uint32_t sgn = static_cast<uint32_t>(static_cast<int32_t>(u) >> 31);
    return (idx ^ sgn) * 8u + t_base;
  }
}

template <int E, int MODE>
__device__ __forceinline__ uint32_t lut_base(const Lut<E>& lut, int lane) {
  if constexpr (E == 16) return smem_u32(&lut.r[0][lane & 15]) - 128u * (0x4B400000u - 15u);
  else if constexpr (MODE == kModeLutI) return smem_u32(lut.i) + 4u * 3073u;
  else return smem_u32(lut.e) + 8u * 1537u;
}

// kModeLutI (256-entry tables): i[bucket256i(q)] + key(q), whose byte 2 is
// the code.  t_base = &i[3073]; the bucket offset is negative for negative q
// (32-bit wrap-around arithmetic).
__device__ __forceinline__ uint32_t lut_int_sum(float q, uint32_t t_base) {
  int32_t off;
  uint32_t key;
  lut_int_index(q, off, key);
  return lds_u32(static_cast<uint32_t>(off) * 4u + t_base) + key;
}

// Weight of element j within its 16-bit half of the output: a half holds 4
// codes of 4 bits (element order in a byte: high nibble first) or 2 codes of
// 8 bits, little-endian.
template <int E>
__device__ __forceinline__ constexpr float half_weight(int j) {
  if constexpr (E == 16) {
    constexpr float w4[4] = {16.0f, 1.0f, 4096.0f, 256.0f};
    return w4[j & 3];
  } else {
    return (j & 1) ? 256.0f : 1.0f;
  }
}

// Fast path: the block's reciprocal is valid for Markstein's form and the
// codebook has a bucket table.  Two elements per packed division and bucket
// computation; one 64-bit table load per element (conflict-free for 16-entry
// tables: each lane reads its own copy).
//  kModeLut:  code = q >= t ? code1 : code0, inserted with a bit-field insert.
//  kModeLutF: H = sat(fma(q, 2^60, K)) is exactly [q >= t]; code = C + H is
//             accumulated in fp32 into 16-bit halves (2^23 + sum of
//             code * weight, every value an exact integer below 2^24; the
//             first element of a half brings the 2^23), and the halves' low
//             bytes are merged with one byte permute per word.
//  kModeLutI (256-entry tables): code = byte 2 of i[b] + key(q)
//             (bq_search.cuh); byte permutes gather four codes into a word.
//  PREW: the elements come already widened to fp32 in xe (quantize_tile).
//  REMAP (16-entry tables like FP4, whose +-0 pair makes one step of two):
//             the table holds ranks of the distinct values, which step by
//             one; each nibble >= 8 then gets 1 added (ranks 8..14 -> codes
//             9..15), three instructions per 8 codes.
template <int DT, int E, int MODE, bool REMAP, bool PREW = false>
__device__ __forceinline__ void encode_fast(const uint32_t (&w)[kThreadWords], const BlockScale& sc,
                                            uint32_t t_base, uint32_t (&ow)[QOut<DT, E>::NW],
                                            const float* xe = nullptr) {
  using O = QOut<DT, E>;
  constexpr int NH = 2 * O::NW;                 // 16-bit halves
  constexpr int PER_HALF = O::EPT / NH;         // elements per half (4 or 2)
  float hacc[NH];
  uint32_t pair[2 * O::NW];  // kModeLutI: codes of elements 2i, 2i+1 in bytes 0, 1
#pragma unroll
  for (int k = 0; k < O::NW; ++k) ow[k] = 0u;
#pragma unroll
  for (int i = 0; i < O::EPT / 2; ++i) {
    float q0, q1;
    if constexpr (DT == kF32)
      div_fast2(tile_elem<DT>(w, 2 * i), tile_elem<DT>(w, 2 * i + 1), sc, q0, q1);
    else
      div_fast2_2term(PREW ? xe[2 * i] : tile_elem<DT>(w, 2 * i),
                      PREW ? xe[2 * i + 1] : tile_elem<DT>(w, 2 * i + 1), sc, q0, q1);
    if constexpr (MODE == kModeLutI) {
      static_assert(E == 256, "integer select is built for 256-entry tables only");
      pair[i] = __byte_perm(lut_int_sum(q0, t_base), lut_int_sum(q1, t_base), 0x0062);
      continue;
    }
    float b0 = q0, b1 = q1;
    if constexpr (E == 16)
      unpack2(fma2(pack2(q0, q1), pack2(15.0f, 15.0f), pack2(12582912.0f, 12582912.0f)), b0, b1);
    const uint2 e0 = lds_u64(lut_addr<E>(b0, t_base));
    const uint2 e1 = lds_u64(lut_addr<E>(b1, t_base));
    const int j0 = 2 * i, j1 = 2 * i + 1;
    if constexpr (MODE == kModeLutF) {
      const float h0 = fma_sat(q0, kSelScale, __uint_as_float(e0.x));
      const float h1 = fma_sat(q1, kSelScale, __uint_as_float(e1.x));
      float& a0 = hacc[j0 / PER_HALF];
      a0 = __fmaf_rn(__uint_as_float(e0.y), half_weight<E>(j0),
                     j0 % PER_HALF == 0 ? 8388608.0f : a0);  // 2^23 enters once
      a0 = __fmaf_rn(h0, half_weight<E>(j0), a0);
      float& a1 = hacc[j1 / PER_HALF];
      a1 = __fmaf_rn(__uint_as_float(e1.y), half_weight<E>(j1), a1);
      a1 = __fmaf_rn(h1, half_weight<E>(j1), a1);
    } else {
      const uint32_t c0 = q0 >= __uint_as_float(e0.x) ? (e0.y >> 8) : e0.y;
      const uint32_t c1 = q1 >= __uint_as_float(e1.x) ? (e1.y >> 8) : e1.y;
      ow[j0 / O::PER_WORD] = bfi(c0, ow[j0 / O::PER_WORD], code_pos<E>(j0), O::L);
      ow[j1 / O::PER_WORD] = bfi(c1, ow[j1 / O::PER_WORD], code_pos<E>(j1), O::L);
    }
  }
  if constexpr (MODE == kModeLutI) {
#pragma unroll
    for (int k = 0; k < O::NW; ++k) ow[k] = __byte_perm(pair[2 * k], pair[2 * k + 1], 0x5410);
  }
  if constexpr (MODE == kModeLutF) {
#pragma unroll
    for (int k = 0; k < O::NW; ++k)
      ow[k] = __byte_perm(__float_as_uint(hacc[2 * k]), __float_as_uint(hacc[2 * k + 1]), 0x5410);
    if constexpr (E == 16) {
      // ranks 8..14 -> codes 9..15: add bit 3 of every nibble to that nibble
      if constexpr (REMAP) {
#pragma unroll
        for (int k = 0; k < O::NW; ++k) ow[k] += (ow[k] >> 3) & 0x11111111u;
      }
    }
  }
}

// Any table form, any block: IEEE division where Markstein's form is not
// valid, clamped lookups.  Exact for every finite input, and never indexes
// outside the tables for any input.  Inlined (an out-of-line call would move
// the thread's registers through local memory on every tile).
template <int DT, int E, int MODE>
__device__ __forceinline__ void encode_safe(const uint32_t (&w)[kThreadWords], const BlockScale& sc,
                                            const TableSmem& tab, const Lut<E>& lut,
                                            uint32_t (&ow)[QOut<DT, E>::NW]) {
  using O = QOut<DT, E>;
#pragma unroll
  for (int k = 0; k < O::NW; ++k) ow[k] = 0u;
#pragma unroll
  for (int j = 0; j < O::EPT; ++j) {
    const float x = tile_elem<DT>(w, j);
    const float xn = fabsf(x) < sc.theta ? div_exact(x, sc.A) : div_fast(x, sc);
    const uint32_t c = search<E, MODE>(xn, tab, lut);
    ow[j / O::PER_WORD] |= (c & ((1u << O::L) - 1u)) << code_pos<E>(j);
  }
}

// --------------------------------------------------- one tile (consumer) --

template <int DT, int E, int TPB, int MODE, bool REMAP>
__device__ __forceinline__ bool quantize_tile(QSmem<E>& s, const QParams& p, uint32_t tile,
                                              int st, uint32_t par, int ct, uint32_t t_base) {
  using O = QOut<DT, E>;
  constexpr int TE = kTileBytes / ElemBytes<DT>::value;
  constexpr int BPT = kQConsumers / TPB;
  const int lane = ct & 31;

  // warp-uniform: if any lane gives up, the whole warp leaves together
  if (!__all_sync(0xffffffffu, mbar_wait_bounded(&s.full[st], par))) {
    if (lane == 0) record_fault(1u);
    return false;
  }

  // four 16-byte chunks of row ct/2, physical chunk = logical ^ (row % 8)
  uint32_t w[kThreadWords];
  {
    const int r = ct >> 1;
    const uint8_t* row = s.stage[st] + r * 128;
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const int chunk = ((ct & 1) << 2) + k;
      const uint4 v = *reinterpret_cast<const uint4*>(row + ((chunk ^ (r & 7)) << 4));
      w[4 * k + 0] = v.x; w[4 * k + 1] = v.y; w[4 * k + 2] = v.z; w[4 * k + 3] = v.w;
    }
  }

  float A;
  // 16-bit inputs, blocks of 4 to 16 threads: widen the elements to fp32
  // before the shuffle tree, so that the compiler can place that independent
  // work between the tree's dependent steps (bf16 / fp16 NF4 blocksize 256,
  // 1 GiB: 229.8 -> 225.6 / 221.4 us; blocks of 2 threads gained nothing)
  constexpr bool PREW_T = DT != kF32 && TPB >= 4 && TPB < 32;
  float xe[O::EPT];
  if constexpr (kStatsWarp<TPB>) {
    // the statistics warp's absmax of this thread's block
    if (!__all_sync(0xffffffffu, mbar_wait_bounded(&s.stats[st], par))) {
      if (lane == 0) record_fault(1u);
      return false;
    }
    A = s.tamax[st][ct / TPB];
    fence_proxy_async_smem();  // the stage's next fill is an async-proxy (TMA) write
    __syncwarp();
    if (lane == 0) mbar_arrive(&s.empty[st]);  // data is in registers: free the stage
  } else {
    // thread-local absmax, NaN-propagating
    float amax;
    if constexpr (DT == kF32) {
      amax = fabsf(__uint_as_float(w[0]));
#pragma unroll
      for (int j = 1; j < kThreadWords; ++j) amax = max_nan(amax, fabsf(__uint_as_float(w[j])));
    } else {
      uint32_t m2 = amax2<DT>(w[0], w[1]);
#pragma unroll
      for (int j = 2; j < kThreadWords; ++j) m2 = amax2<DT>(m2, w[j]);
      amax = max_nan(fabsf(widen_pair_elem<DT>(m2, 0)), fabsf(widen_pair_elem<DT>(m2, 1)));
    }
    fence_proxy_async_smem();  // the stage's next fill is an async-proxy (TMA) write
    __syncwarp();
    if (lane == 0) mbar_arrive(&s.empty[st]);  // data is in registers: free the stage

    float m = amax;
    if constexpr (PREW_T) {
#pragma unroll
      for (int j = 0; j < O::EPT; ++j) xe[j] = tile_elem<DT>(w, j);
    }
    (void)xe;
    if constexpr (TPB == 32) {
      // |x| >= 0 (or a NaN with the sign clear): the bits order as unsigned
      // integers, NaN above +inf, so one integer max reduces the warp
      m = __uint_as_float(__reduce_max_sync(0xffffffffu, __float_as_uint(m)));
    } else if constexpr (TPB == 16) {
      // the same integer reduction over each half-warp (the two halves are
      // reduced one after the other, which for 2 groups still beats a 4-level
      // shuffle tree: 1 GiB dyn8 bf16 blocksize 512 327.9 -> 313.6 us, fp32
      // blocksize 256 225.7 -> 215.4 us; for 4 or more groups it did not)
      const uint32_t gmask = 0xffffu << (lane & 16);
      m = __uint_as_float(__reduce_max_sync(gmask, __float_as_uint(m)));
    } else if constexpr (TPB > 1) {
#pragma unroll
      for (int off = 1; off < TPB; off <<= 1) m = max_nan(m, __shfl_xor_sync(0xffffffffu, m, off));
    }
    A = m;
    if (ct % TPB == 0) p.absmax[static_cast<int64_t>(tile) * BPT + ct / TPB] = A;
  }

  uint32_t ow[O::NW];
  // bucket path: the block's reciprocal is valid for Markstein's form (the
  // per-element condition is not needed, see div_fast); NaN fails both tests
  constexpr bool kBucket = MODE == kModeLut || MODE == kModeLutF || MODE == kModeLutI;
  const bool fast = kBucket && (A == 0.0f || (A >= 0x1p-60f && A <= 0x1p60f));
  if (fast)
    encode_fast<DT, E, kBucket ? MODE : kModeLut, REMAP, PREW_T>(
        w, DT == kF32 ? make_scale_fast(A) : make_scale_fast_2term(A), t_base, ow, xe);
  else encode_safe<DT, E, MODE>(w, make_scale(A), s.tab, s.lut, ow);

  const int64_t e0 = static_cast<int64_t>(tile) * TE + static_cast<int64_t>(ct) * O::EPT;
  uint8_t* dst = p.out + (E == 16 ? e0 / 2 : e0);
#pragma unroll
  for (int k = 0; k < O::NW; k += 4) {
    if constexpr (O::NW >= 4) {
      *reinterpret_cast<uint4*>(dst + 4 * k) = make_uint4(ow[k], ow[k + 1], ow[k + 2], ow[k + 3]);
    }
  }
  if constexpr (O::NW == 2) *reinterpret_cast<uint2*>(dst) = make_uint2(ow[0], ow[1]);
  return true;
}

// ------------------------------------------ one block per warp (generic) --

template <int DT, int E, int MODE>
__device__ void quantize_block_generic(const QParams& p, const QSmem<E>& s, int64_t b, int lane) {
  const int64_t lo = b * p.bs;
  const int64_t hi = min(p.n, lo + p.bs);
  float m = 0.0f;
  for (int64_t i = lo + lane; i < hi; i += 32) m = max_nan(m, fabsf(load_elem<DT>(p.x, i)));
#pragma unroll
  for (int off = 16; off >= 1; off >>= 1) m = max_nan(m, __shfl_xor_sync(0xffffffffu, m, off));
  const float A = m;
  if (lane == 0) p.absmax[b] = A;
  if constexpr (E == 16) {
    for (int64_t q = lo / 2 + lane; q < (hi + 1) / 2; q += 32) {
      const int64_t i0 = 2 * q;
      const uint32_t c0 = search<E, MODE>(div_exact(load_elem<DT>(p.x, i0), A), s.tab, s.lut);
      uint32_t c1 = 0;
      if (i0 + 1 < hi) c1 = search<E, MODE>(div_exact(load_elem<DT>(p.x, i0 + 1), A), s.tab, s.lut);
      p.out[q] = static_cast<uint8_t>(((c0 & 15u) << 4) | (c1 & 15u));
    }
  } else {
    for (int64_t i = lo + lane; i < hi; i += 32)
      p.out[i] = static_cast<uint8_t>(search<E, MODE>(div_exact(load_elem<DT>(p.x, i), A), s.tab, s.lut));
  }
}

// ---------------------------------------------------- statistics warp ----

// Absmax of the quantization blocks b of each tile with b % NSW == sw (TPB >
// 32: a block is TPB / 2 >= 32 whole 128-byte rows, one to four blocks per
// tile), written to the stage's tamax slots and to global memory; then the
// stage's stats mbarrier (NSW arrivals) is signalled and the stage released
// like a consumer warp does.
// Step k reads bytes [512 k, 512 k + 512) of the stage, lane l the 16 bytes at
// 512 k + 16 l (four whole rows, so the 128-byte swizzle, a permutation within
// each row, does not matter, and the warp's load is free of bank conflicts);
// a block is TPB / 8 consecutive steps.  |x| is kept as bits: for values >= 0
// (and NaN, sign cleared) the unsigned order is the float order with NaN above
// +inf, so the warp's maximum is one integer reduction.
template <int DT, int E, int TPB>
__device__ void stats_main(QSmem<E>& s, const QParams& p, int lane, int sw) {
  constexpr int NSW = kNumStats<DT, E, TPB>;
  constexpr int BPT = kQConsumers / TPB;
  constexpr int STEPS = TPB / 8;   // 512-byte steps per block
  static_assert(BPT <= kQMaxTileBlocks && STEPS * BPT == kTileBytes / 512, "tile split");
  pdl_wait();  // absmax is written to global memory
  const uint32_t ntiles = static_cast<uint32_t>(p.full_tiles);
  uint32_t iter = 0;
  for (uint32_t tile = blockIdx.x; tile < ntiles; tile += gridDim.x, ++iter) {
    const int st = static_cast<int>(iter % kStages);
    const uint32_t par = (iter / kStages) & 1u;
    if (!__all_sync(0xffffffffu, mbar_wait_bounded(&s.full[st], par))) {
      if (lane == 0) record_fault(1u);
      break;
    }
    const uint8_t* src = s.stage[st] + 16 * lane;
#pragma unroll
    for (int b = 0; b < BPT; ++b) {
      if (b % NSW != sw) continue;
      uint32_t mb;  // bits of this lane's max |x| over the block
      if constexpr (DT == kF32) {
        float m = 0.0f;
#pragma unroll 8
        for (int k = 0; k < STEPS; ++k) {
          const uint4 v = *reinterpret_cast<const uint4*>(src + 512 * (b * STEPS + k));
          m = max_nan(m, max_nan(max_nan(fabsf(__uint_as_float(v.x)), fabsf(__uint_as_float(v.y))),
                                 max_nan(fabsf(__uint_as_float(v.z)), fabsf(__uint_as_float(v.w)))));
        }
        mb = __float_as_uint(m);
      } else {
        uint32_t m2 = 0u;
#pragma unroll 8
        for (int k = 0; k < STEPS; ++k) {
          const uint4 v = *reinterpret_cast<const uint4*>(src + 512 * (b * STEPS + k));
          m2 = amax2<DT>(m2, amax2<DT>(amax2<DT>(v.x, v.y), amax2<DT>(v.z, v.w)));
        }
        mb = __float_as_uint(max_nan(fabsf(widen_pair_elem<DT>(m2, 0)),
                                     fabsf(widen_pair_elem<DT>(m2, 1))));
      }
      const float A = __uint_as_float(__reduce_max_sync(0xffffffffu, mb));
      if (lane == 0) {
        s.tamax[st][b] = A;
        p.absmax[static_cast<int64_t>(tile) * BPT + b] = A;
      }
    }
    if (lane == 0) mbar_arrive(&s.stats[st]);  // releases the tamax writes
    fence_proxy_async_smem();  // the stage's next fill is an async-proxy (TMA) write
    __syncwarp();
    if (lane == 0) mbar_arrive(&s.empty[st]);
  }
}

// ------------------------------------------------------------- kernel -----

template <int DT, int E, int TPB, int MODE, bool REMAP = false>
__device__ __forceinline__ void consumer_main(QSmem<E>& s, const QParams& p, int ct) {
  constexpr int BPT = kQConsumers / TPB;
  const uint32_t t_base = lut_base<E, MODE>(s.lut, ct & 31);
  const uint32_t ntiles = static_cast<uint32_t>(p.full_tiles);  // < 2^24 (host check)
  uint32_t iter = 0;
  for (uint32_t tile = blockIdx.x; tile < ntiles; tile += gridDim.x, ++iter) {
    const int st = static_cast<int>(iter % kStages);
    const uint32_t par = (iter / kStages) & 1u;
    if (!quantize_tile<DT, E, TPB, MODE, REMAP>(s, p, tile, st, par, ct, t_base)) break;
  }
  // what the tiles did not cover: one quantization block per warp
  const int lane = ct & 31, cw = ct >> 5;
  const int64_t nwarps = static_cast<int64_t>(gridDim.x) * kQConsumerWarps;
  for (int64_t b = p.full_tiles * BPT + static_cast<int64_t>(blockIdx.x) * kQConsumerWarps + cw;
       b < p.nb; b += nwarps)
    quantize_block_generic<DT, E, MODE>(p, s, b, lane);
}

template <int DT, int E, int TPB>
__global__ void __launch_bounds__(q_threads<DT, E, TPB>(), 2)
    quantize_kernel(const __grid_constant__ CUtensorMap tmap, const QParams p) {
  extern __shared__ uint8_t smem_raw[];
  QSmem<E>& s = *reinterpret_cast<QSmem<E>*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  constexpr bool SW = kStatsWarp<TPB>;
  constexpr int NSW = kNumStats<DT, E, TPB>;

  if (threadIdx.x == 0) {
    for (int i = 0; i < kStages; ++i) {
      mbar_init(&s.full[i], 1);
      mbar_init(&s.empty[i], kQConsumerWarps + NSW);
      mbar_init(&s.stats[i], NSW > 0 ? NSW : 1);
    }
    fence_mbar_init();
  }
  pdl_release();
  __syncthreads();

  // Under programmatic dependent launch this CTA may start while earlier
  // kernels on the stream still run.  The search tables are built from the
  // codebook before waiting for them, so that the build overlaps their tail;
  // after the wait the codebook is read again and, if any entry changed (an
  // earlier kernel wrote it), the tables are built once more.  The input is
  // read and the outputs are written only after the wait.
  if (warp == 0) {
    pdl_wait();
    if (lane == 0 && p.full_tiles > 0) {
      int64_t iter = 0;
      for (int64_t tile = blockIdx.x; tile < p.full_tiles; tile += gridDim.x, ++iter) {
        const int st = static_cast<int>(iter % kStages);
        if (iter >= kStages) {
          const uint32_t par = static_cast<uint32_t>(((iter / kStages) & 1) ^ 1);
          if (!mbar_wait_bounded(&s.empty[st], par)) {
            record_fault(2u);
            break;
          }
        }
        if (test_skip_tile(tile)) continue;  // fault-path test builds only
        mbar_arrive_expect_tx(&s.full[st], kTileBytes);
        tma_load_2d(s.stage[st], &tmap, 0, static_cast<int32_t>(tile * kTileRows), &s.full[st]);
      }
      // every copy issued must have landed before the CTA may exit
      for (int64_t j = iter > kStages ? iter - kStages : 0; j < iter; ++j)
        (void)mbar_wait_bounded(&s.full[j % kStages], static_cast<uint32_t>((j / kStages) & 1));
    }
    return;
  }
  if constexpr (SW) {
    if (warp >= 1 && warp <= NSW) {
      stats_main<DT, E, TPB>(s, p, lane, warp - 1);
      return;
    }
  }

  const int ct = threadIdx.x - 32 * (1 + NSW);
  build_search<E, kQConsumers>(s.tab, s.lut, p.code, ct);
  pdl_wait();
  // the tables stand only if the codebook, read at L2 after the wait, still
  // holds the bits they were built from
  const bool stale = ct < E && __float_as_uint(__ldcg(p.code + ct)) != __float_as_uint(s.tab.c[ct]);
  if (named_sync_or(1, kQConsumers, stale)) build_search<E, kQConsumers>(s.tab, s.lut, p.code, ct);
  const int mode = s.tab.mode;
  // REMAP: FP4-like 16-entry tables, float select over ranks (bq_search.cuh)
  if (mode == kModeLutF && E == 16 && s.tab.remap8)
    consumer_main<DT, E, TPB, kModeLutF, E == 16>(s, p, ct);
  else if (mode == kModeLutF) consumer_main<DT, E, TPB, kModeLutF>(s, p, ct);
  else if (E == 256 && mode == kModeLutI) consumer_main<DT, E, TPB, E == 256 ? kModeLutI : kModeLutF>(s, p, ct);
  else if (mode == kModeLut) consumer_main<DT, E, TPB, kModeLut>(s, p, ct);
  else if (mode == kModeBsearch) consumer_main<DT, E, TPB, kModeBsearch>(s, p, ct);
  else consumer_main<DT, E, TPB, kModeScan>(s, p, ct);
}

}  // namespace bq
