// bq_quantize.cuh - blockwise absmax codebook quantization (sm_100a).
//
// Method: "bitsandbytes PR #2052" (General8 / FP4 / NF4 blockwise
// quantization, block sizes 32..4096, full blocks and tails, FP16 / BF16 /
// FP32 inputs).  Per block: absmax, xn = x / absmax (IEEE fp32), nearest code
// (lowest index on ties), codes packed two per byte high nibble first
// (16-entry tables) or one per byte (256-entry tables).
//
// Kernel design.  A persistent grid (<= 2 CTAs per SM) of 288-thread CTAs: one
// producer warp streams 16 KiB input tiles (128 rows of 128 B) into a 4-stage
// shared-memory ring with 2-D TMA loads (128-byte swizzle, no multicast), and
// 8 consumer warps process each tile.  Consumer thread t owns 64 contiguous
// bytes of the tile (row t/2, half t%2), read with four conflict-free 16-byte
// shared loads thanks to the swizzle.  A quantization block therefore spans
// TPB = blocksize * elem_bytes / 64 consecutive threads: its absmax is a
// shuffle-xor tree over TPB lanes, plus a shared-memory step across warps when
// TPB > 32 (blocksize 4096 in 16-bit types, 2048+ in fp32).  The stage is
// released right after the absmax pass (the data is in registers by then).
// Normalisation uses the per-block reciprocal with Markstein's correction
// (exact), the search the bucket table of bq_search.cuh, and each thread
// stores its packed codes with one or two 16-byte stores.  Bytes of the input
// that do not fill a whole tile, and every input that is not 16-byte aligned,
// are handled one block per warp from global memory with the same arithmetic.
#pragma once

#include "bq_search.cuh"

namespace bq {

constexpr int kQThreads = 288;    // warp 0: producer; warps 1..8: consumers
constexpr int kQConsumers = 256;
constexpr int kTileBytes = 16384;
constexpr int kTileRows = 128;    // rows of 128 bytes
constexpr int kStages = 4;

template <int E>
struct QSmem {
  uint8_t stage[kStages][kTileBytes];  // 1024-byte aligned (128B swizzle)
  uint64_t full[kStages];
  uint64_t empty[kStages];
  float red[2][8];
  int cabort[2];   // per tile-iteration parity: a consumer gave up waiting
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

// ------------------------------------------------- one element -> code ----

template <int DT, int EPT>
__device__ __forceinline__ float tile_elem(const uint32_t (&w)[16], int j) {
  if constexpr (DT == kF32) return __uint_as_float(w[j]);
  else return widen_pair_elem<DT>(w[j >> 1], j & 1);
}

// Codes of a thread's EPT elements packed into words: 4-bit codes put element
// 2i in the high nibble of byte i; 8-bit codes one per byte.
template <int DT, int E, int MODE, int EPT, bool SLOW>
__device__ __forceinline__ void encode_thread(const uint32_t (&w)[16], const BlockScale& sc,
                                              const TableSmem& tab, const Lut<E>& lut,
                                              uint32_t (&ow)[E == 16 ? EPT / 8 : EPT / 4],
                                              bool& any_small) {
  constexpr int NW = E == 16 ? EPT / 8 : EPT / 4;
#pragma unroll
  for (int k = 0; k < NW; ++k) ow[k] = 0;
  bool small = false;
#pragma unroll
  for (int j = 0; j < EPT; ++j) {
    const float x = tile_elem<DT, EPT>(w, j);
    float xn;
    if constexpr (SLOW) {
      xn = fabsf(x) < sc.theta ? div_exact(x, sc.A) : div_fast(x, sc);
    } else {
      xn = div_fast(x, sc);
      if constexpr (DT != kF16) small |= fabsf(x) < sc.theta;
    }
    const uint32_t c = search<E, MODE>(xn, tab, lut);
    if constexpr (E == 16) {
      ow[j >> 3] |= c << ((((j & 7) >> 1) << 3) + ((j & 1) ? 0 : 4));
    } else {
      ow[j >> 2] |= c << ((j & 3) << 3);
    }
  }
  any_small = small;
}

// --------------------------------------------------- one tile (consumer) --

template <int DT, int E, int TPB, int MODE>
__device__ __forceinline__ bool quantize_tile(QSmem<E>& s, const QParams& p, int64_t tile,
                                              int st, uint32_t par, int64_t iter, int ct) {
  constexpr int EB = ElemBytes<DT>::value;
  constexpr int EPT = 64 / EB;
  constexpr int TE = kTileBytes / EB;
  constexpr int BPT = kQConsumers / TPB;
  const int lane = ct & 31, cw = ct >> 5;

  const bool ok = mbar_wait_bounded(&s.full[st], par);
  if (!ok) {
    if (lane == 0) record_fault(1u);
    s.cabort[iter & 1] = 1;
  }

  // four 16-byte chunks of row ct/2, physical chunk = logical ^ (row % 8)
  uint32_t w[16];
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
  float m = 0.0f;
#pragma unroll
  for (int j = 0; j < EPT; ++j) m = fmaxf(m, fabsf(tile_elem<DT, EPT>(w, j)));
  __syncwarp();
  if (lane == 0) mbar_arrive(&s.empty[st]);  // data is in registers: free the stage

  bool abort_now = !ok;
  if constexpr (TPB > 1 && TPB <= 32) {
#pragma unroll
    for (int off = 1; off < TPB; off <<= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, off));
  } else if constexpr (TPB > 32) {
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, off));
    constexpr int WPB = TPB / 32;
    const int pb = static_cast<int>(iter & 1);
    if (lane == 0) s.red[pb][cw] = m;
    named_sync(1, kQConsumers);
    const int g0 = (cw / WPB) * WPB;
    m = s.red[pb][g0];
#pragma unroll
    for (int i = 1; i < WPB; ++i) m = fmaxf(m, s.red[pb][g0 + i]);
    // set before this barrier by any warp that gave up on this tile; the slot
    // of the other parity may already be written by a warp one tile ahead
    abort_now = *reinterpret_cast<volatile int*>(&s.cabort[iter & 1]) != 0;
  }
  const float A = m;
  if (abort_now) return false;

  const int64_t e0 = tile * TE + static_cast<int64_t>(ct) * EPT;
  if (ct % TPB == 0) p.absmax[tile * BPT + ct / TPB] = A;

  const BlockScale sc = make_scale(A);
  constexpr int NW = E == 16 ? EPT / 8 : EPT / 4;
  uint32_t ow[NW];
  bool any_small;
  encode_thread<DT, E, MODE, EPT, false>(w, sc, s.tab, s.lut, ow, any_small);
  if (any_small) encode_thread<DT, E, MODE, EPT, true>(w, sc, s.tab, s.lut, ow, any_small);

  uint8_t* dst = p.out + (E == 16 ? e0 / 2 : e0);
  if constexpr (NW == 2) {
    *reinterpret_cast<uint2*>(dst) = make_uint2(ow[0], ow[1]);
  } else {
#pragma unroll
    for (int k = 0; k < NW; k += 4)
      *reinterpret_cast<uint4*>(dst + 4 * k) = make_uint4(ow[k], ow[k + 1], ow[k + 2], ow[k + 3]);
  }
  return true;
}

// ------------------------------------------ one block per warp (generic) --

template <int DT, int E, int MODE>
__device__ void quantize_block_generic(const QParams& p, const QSmem<E>& s, int64_t b, int lane) {
  const int64_t lo = b * p.bs;
  const int64_t hi = min(p.n, lo + p.bs);
  float m = 0.0f;
  for (int64_t i = lo + lane; i < hi; i += 32) m = fmaxf(m, fabsf(load_elem<DT>(p.x, i)));
#pragma unroll
  for (int off = 16; off >= 1; off >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, off));
  const float A = m;
  if (lane == 0) p.absmax[b] = A;
  if constexpr (E == 16) {
    for (int64_t q = lo / 2 + lane; q < (hi + 1) / 2; q += 32) {
      const int64_t i0 = 2 * q;
      const uint32_t c0 = search<E, MODE>(div_exact(load_elem<DT>(p.x, i0), A), s.tab, s.lut);
      uint32_t c1 = 0;
      if (i0 + 1 < hi) c1 = search<E, MODE>(div_exact(load_elem<DT>(p.x, i0 + 1), A), s.tab, s.lut);
      p.out[q] = static_cast<uint8_t>((c0 << 4) | c1);
    }
  } else {
    for (int64_t i = lo + lane; i < hi; i += 32)
      p.out[i] = static_cast<uint8_t>(search<E, MODE>(div_exact(load_elem<DT>(p.x, i), A), s.tab, s.lut));
  }
}

// ------------------------------------------------------------- kernel -----

template <int DT, int E, int TPB, int MODE>
__device__ __forceinline__ void consumer_main(QSmem<E>& s, const QParams& p, int ct) {
  constexpr int EB = ElemBytes<DT>::value;
  constexpr int BPT = kQConsumers / TPB;
  int64_t iter = 0;
  for (int64_t tile = blockIdx.x; tile < p.full_tiles; tile += gridDim.x, ++iter) {
    const int st = static_cast<int>(iter % kStages);
    const uint32_t par = static_cast<uint32_t>((iter / kStages) & 1);
    if (!quantize_tile<DT, E, TPB, MODE>(s, p, tile, st, par, iter, ct)) break;
  }
  (void)EB;
  // what the tiles did not cover: one quantization block per warp
  const int lane = ct & 31, cw = ct >> 5;
  const int64_t nwarps = static_cast<int64_t>(gridDim.x) * (kQConsumers / 32);
  for (int64_t b = p.full_tiles * BPT + static_cast<int64_t>(blockIdx.x) * (kQConsumers / 32) + cw;
       b < p.nb; b += nwarps)
    quantize_block_generic<DT, E, MODE>(p, s, b, lane);
}

template <int DT, int E, int TPB>
__global__ void __launch_bounds__(kQThreads, 2)
    quantize_kernel(const __grid_constant__ CUtensorMap tmap, const QParams p) {
  extern __shared__ uint8_t smem_raw[];
  QSmem<E>& s = *reinterpret_cast<QSmem<E>*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int i = 0; i < kStages; ++i) {
      mbar_init(&s.full[i], 1);
      mbar_init(&s.empty[i], kQConsumers / 32);
    }
    s.cabort[0] = 0;
    s.cabort[1] = 0;
    fence_mbar_init();
  }
  __syncthreads();

  if (warp == 0) {
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
        mbar_arrive_expect_tx(&s.full[st], kTileBytes);
        tma_load_2d(s.stage[st], &tmap, 0, static_cast<int32_t>(tile * kTileRows), &s.full[st]);
      }
      // every copy issued must have landed before the CTA may exit
      for (int64_t j = iter > kStages ? iter - kStages : 0; j < iter; ++j)
        (void)mbar_wait_bounded(&s.full[j % kStages], static_cast<uint32_t>((j / kStages) & 1));
    }
    return;
  }

  const int ct = threadIdx.x - 32;
  build_search<E>(s.tab, s.lut, p.code, ct);
  const int mode = s.tab.mode;
  if (mode == kModeLut) consumer_main<DT, E, TPB, kModeLut>(s, p, ct);
  else if (mode == kModeBsearch) consumer_main<DT, E, TPB, kModeBsearch>(s, p, ct);
  else consumer_main<DT, E, TPB, kModeScan>(s, p, ct);
}

}  // namespace bq
