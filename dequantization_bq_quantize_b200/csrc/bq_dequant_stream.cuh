// bq_dequant_stream.cuh - blockwise dequantization with the code stream
// staged through shared memory (sm_100a).
//
// Same result as dequant_kernel (bq_dequant.cuh): y_i = narrow(RN(code[idx_i]
// * absmax[i / blocksize])), the inverse map of "bitsandbytes PR #2052".
//
// Why a second kernel.  Dequantization writes about four times the bytes it
// reads.  In dequant_kernel every warp loads its codes and scales, waits for
// them, decodes and stores, so each iteration's stores wait behind the
// global-load latency of its own loads: at n = 2^29 bf16 it takes 254 us,
// and without any loads the same stores take 158 us.  Here the loads run
// ahead: a persistent grid of 544-thread CTAs (3 per SM), one producer lane
// streaming each tile's codes (4 KiB for 4-bit, 8 KiB for 8-bit codes of
// 8192 elements) and its slice of absmax into a 4-stage shared-memory ring
// with 1-D bulk copies (cp.async.bulk, no multicast) completed by mbarrier
// transaction counts, and 16 consumer warps decoding from shared memory.  A
// consumer warp owns 64 consecutive 16-byte output chunks of the tile, so its
// two stores per lane are 1 KiB of contiguous output, and decodes with a
// per-lane copy of the table (below), free of bank conflicts.  The warps
// stall on the global store queue: 48 store-issuing warps per SM instead of
// 32 (8 consumer warps, 4 CTAs per SM) took the kernel in the benchmark step
// from 237.6 to 232.2 us at n = 2^29.  A consumer releases a stage only after
// an async-proxy fence: the stage's next fill is a bulk copy, which the
// mbarrier release / acquire alone does not order after the consumer's plain
// shared-memory loads (without the fence, a few warps per thousand round
// trips decoded with the next tile's scales).
//
// Used for 4-bit codes with plain statistics when codes, absmax and y are
// 16-byte aligned: blocksize <= 2048 streams the tile's absmax slice (a whole
// number of 16-byte units) with the codes, blocksize 4096 has the producer
// lane copy the tile's two scales (ADIRECT); the elements after the last
// whole tile are done one per thread from global memory.  (The template also covers 8-bit
// codes, which measured faster on dequant_kernel.)  Every mbarrier wait gives
// up after a bounded time, sets a bit of the device fault word (4: consumer,
// 8: producer) and leaves the kernel instead of hanging.
#pragma once

#include "bq_dequant.cuh"

namespace bq {

constexpr int kSTile = 8192;                          // elements per tile
constexpr int kSStages = 4;
constexpr int kSConsumerWarps = 16;
constexpr int kSThreads = 32 * (kSConsumerWarps + 1);

// The decode table is replicated per lane so that its lookups never conflict
// on banks (the codes of normal data are close to equiprobable, so a warp's
// lookups hit random entries): 4-bit codes read 8-byte pairs, copy s = lane %
// 16 of pair b at tr + 128 b + 8 s (one 128-byte row per pair, copy s in bank
// pair s); 8-bit codes read 4-byte values, copy l = lane of value b at
// tr + 128 b + 4 l.  32 KiB either way.  At n = 2^29 bf16 NF4 inside the
// benchmark step: 251 us (dequant_kernel) -> 236 us.
template <int E>
struct SSmem {
  static constexpr int CODE_BYTES = E == 16 ? kSTile / 2 : kSTile;
  uint8_t codes[kSStages][CODE_BYTES];                 // 16-byte aligned
  float amax[kSStages][kSTile / 32];                   // blocksize >= 32; NESTED:
                                                       // the statistics codes as bytes
  uint64_t full[kSStages];
  uint64_t empty[kSStages];
  float code[E];
  float code2[256];                                    // NESTED only
  float tr[256 * 32];
};

template <int E>
constexpr size_t ssmem_bytes() { return sizeof(SSmem<E>) + 128; }

template <int QB>
__device__ __forceinline__ uint2 smem_codes(const uint8_t* base, int chunk) {
  if constexpr (QB == 8) return *reinterpret_cast<const uint2*>(base + 8 * chunk);
  else if constexpr (QB == 4) return make_uint2(*reinterpret_cast<const uint32_t*>(base + 4 * chunk), 0u);
  else return make_uint2(*reinterpret_cast<const unsigned short*>(base + 2 * chunk), 0u);
}

// NESTED (compressed statistics): the stage's statistics slot holds the
// tile's statistics codes (one byte per block; blocksize <= 512 keeps them a
// whole number of 16-byte units), and the tile's second-level scale
// (blocksize * blocksize2 >= the tile, so one per tile) comes from global
// memory, fetched a tile ahead.  A_b = RN(code2[qa_b] * absmax2), as in
// dequant_kernel.
//
// ADIRECT (plain statistics, blocksize 4096: a tile's two scales are 8 bytes,
// less than a bulk copy's 16-byte unit): the producer lane reads them with
// plain loads a tile ahead and stores them into the stage's statistics slot
// before its arrive on the stage's full barrier, which releases them to the
// consumers with the codes.  (Each consumer warp reading its own scale from
// global memory measured slower: 246 against 240 us for 1 GiB bf16, the
// loads queueing behind the warps' stores.)
template <int E, int OT, bool NESTED, bool ADIRECT = false>
__global__ void __launch_bounds__(kSThreads) dequant_stream_kernel(const DParams p, int64_t ntiles) {
  static_assert(!(NESTED && ADIRECT), "one statistics form");
  using T = DTraits<E, OT>;
  constexpr int CHUNKS = kSTile / T::CE;                 // 16-byte output chunks per tile
  constexpr int PER_WARP = CHUNKS / kSConsumerWarps;     // 128 or 256
  constexpr int PER_LANE = PER_WARP / 32;                // 4 or 8
  constexpr int CODE_BYTES = SSmem<E>::CODE_BYTES;
  extern __shared__ uint8_t dsmem_raw[];
  SSmem<E>& s = *reinterpret_cast<SSmem<E>*>(
      (reinterpret_cast<uintptr_t>(dsmem_raw) + 127) & ~static_cast<uintptr_t>(127));

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int abs_per_tile = kSTile >> p.bs_log2;
  if (threadIdx.x == 0) {
    for (int i = 0; i < kSStages; ++i) {
      mbar_init(&s.full[i], 1);
      mbar_init(&s.empty[i], kSConsumerWarps);
    }
    fence_mbar_init();
  }
  pdl_release();
  __syncthreads();

  if (warp == kSConsumerWarps) {  // producer
    pdl_wait();  // codes and absmax may be written by the previous kernel
    if (lane == 0) {
      const uint64_t pol = l2_evict_first_policy();
      // ADIRECT: the tile's two scales, read by this lane one tile ahead
      float pa0 = 0.0f, pa1 = 0.0f;
      if constexpr (ADIRECT) {
        if (static_cast<int64_t>(blockIdx.x) < ntiles) {
          pa0 = __ldg(p.absmax + 2 * static_cast<int64_t>(blockIdx.x));
          pa1 = __ldg(p.absmax + 2 * static_cast<int64_t>(blockIdx.x) + 1);
        }
      }
      int64_t iter = 0;
      for (int64_t tile = blockIdx.x; tile < ntiles; tile += gridDim.x, ++iter) {
        const int st = static_cast<int>(iter % kSStages);
        if (iter >= kSStages) {
          const uint32_t par = static_cast<uint32_t>(((iter / kSStages) & 1) ^ 1);
          if (!mbar_wait_bounded(&s.empty[st], par)) {
            record_fault(8u);
            break;
          }
        }
        if (test_skip_tile(tile)) continue;  // fault-path test builds only
        if constexpr (ADIRECT) {
          // plain shared stores, released to the consumers by the arrive below
          s.amax[st][0] = pa0;
          s.amax[st][1] = pa1;
          const int64_t nt = tile + gridDim.x;
          if (nt < ntiles) {
            pa0 = __ldg(p.absmax + 2 * nt);
            pa1 = __ldg(p.absmax + 2 * nt + 1);
          }
        }
        const uint32_t abytes =
            ADIRECT ? 0u : (NESTED ? 1u : 4u) * static_cast<uint32_t>(abs_per_tile);
        mbar_arrive_expect_tx(&s.full[st], CODE_BYTES + abytes);
        bulk_load(s.codes[st], p.q + tile * CODE_BYTES, CODE_BYTES, &s.full[st], pol);
        if constexpr (NESTED)
          bulk_load(s.amax[st], p.qa + tile * abs_per_tile, abytes, &s.full[st], pol);
        else if constexpr (!ADIRECT)
          bulk_load(s.amax[st], p.absmax + tile * abs_per_tile, abytes, &s.full[st], pol);
      }
      // every copy issued must have landed before the CTA may exit
      for (int64_t j = iter > kSStages ? iter - kSStages : 0; j < iter; ++j)
        (void)mbar_wait_bounded(&s.full[j % kSStages], static_cast<uint32_t>((j / kSStages) & 1));
    }
    return;
  }

  // consumers: the codebook (pair table for 4-bit codes), then the tiles
  const int ct = threadIdx.x;  // 0 .. 32 * kSConsumerWarps - 1
  pdl_wait();
  for (int i = ct; i < E; i += 32 * kSConsumerWarps) s.code[i] = p.code[i];
  if constexpr (NESTED)
    for (int i = ct; i < 256; i += 32 * kSConsumerWarps) s.code2[i] = p.code2[i];
  named_sync(1, 32 * kSConsumerWarps);
  if constexpr (E == 16) {
    // entry (b, copy c) = (code[b >> 4], code[b & 15]) at float index 32 b + 2 c
    for (int i = ct; i < 256 * 16; i += 32 * kSConsumerWarps) {
      const int b = i >> 4, c = i & 15;
      s.tr[32 * b + 2 * c] = s.code[b >> 4];
      s.tr[32 * b + 2 * c + 1] = s.code[b & 15];
    }
  } else {
    for (int i = ct; i < 256 * 32; i += 32 * kSConsumerWarps) s.tr[i] = s.code[i >> 5];
  }
  named_sync(1, 32 * kSConsumerWarps);
  const uint32_t t_base = smem_u32(s.tr) + (E == 16 ? 8u * (lane & 15) : 4u * lane);

  uint4* y4 = static_cast<uint4*>(p.y);
  // NESTED: second-level scale of the tile (block index >> bs2_log2 of the
  // tile's first block), loaded one tile ahead
  const int sh2 = p.bs2_log2 + p.bs_log2;
  float a2_next = 0.0f;
  if constexpr (NESTED)
    if (static_cast<int64_t>(blockIdx.x) < ntiles)
      a2_next = __ldg(p.absmax2 + ((static_cast<int64_t>(blockIdx.x) * kSTile) >> sh2));
  int64_t iter = 0;
  for (int64_t tile = blockIdx.x; tile < ntiles; tile += gridDim.x, ++iter) {
    float a2 = 0.0f;
    if constexpr (NESTED) {
      a2 = a2_next;
      const int64_t nt = tile + gridDim.x;
      if (nt < ntiles) a2_next = __ldg(p.absmax2 + ((nt * kSTile) >> sh2));
    }
    const int st = static_cast<int>(iter % kSStages);
    // warp-uniform: if any lane gives up, the whole warp leaves together
    if (!__all_sync(0xffffffffu,
                    mbar_wait_bounded(&s.full[st], static_cast<uint32_t>((iter / kSStages) & 1)))) {
      if (lane == 0) record_fault(4u);
      break;  // the producer gives up too, on the stage this warp never frees
    }
    uint2 c[PER_LANE];
    float A[PER_LANE];
#pragma unroll
    for (int u = 0; u < PER_LANE; ++u) {
      const int ch = warp * PER_WARP + u * 32 + lane;
      c[u] = smem_codes<T::QB>(s.codes[st], ch);
      if constexpr (NESTED) {
        const uint32_t qa = reinterpret_cast<const uint8_t*>(s.amax[st])[(ch * T::CE) >> p.bs_log2];
        A[u] = __fmul_rn(s.code2[qa], a2);
      } else {
        A[u] = s.amax[st][(ch * T::CE) >> p.bs_log2];
      }
    }
    fence_proxy_async_smem();  // the stage's next fill is an async-proxy write
    __syncwarp();
    if (lane == 0) mbar_arrive(&s.empty[st]);  // this warp's part is in registers
    const int64_t first = tile * CHUNKS + warp * PER_WARP + lane;
#pragma unroll
    for (int u = 0; u < PER_LANE; ++u)
      y4[first + u * 32] = decode_chunk<E, OT, 128>(c[u], A[u], t_base);
  }

  // the elements after the last whole tile, one per thread
  const int64_t gtid = static_cast<int64_t>(blockIdx.x) * (32 * kSConsumerWarps) + ct;
  const int64_t gsz = static_cast<int64_t>(gridDim.x) * (32 * kSConsumerWarps);
  for (int64_t i = ntiles * kSTile + gtid; i < p.n; i += gsz) {
    uint32_t idx;
    if constexpr (E == 16) {
      const uint32_t byte = p.q[i >> 1];
      idx = (i & 1) ? (byte & 15u) : (byte >> 4);
    } else {
      idx = p.q[i];
    }
    const int64_t b = i >> p.bs_log2;
    float A;
    if constexpr (NESTED) A = __fmul_rn(s.code2[p.qa[b]], __ldg(p.absmax2 + (b >> p.bs2_log2)));
    else A = __ldg(p.absmax + b);
    store_elem<OT>(p.y, i, __fmul_rn(s.code[idx], A));
  }
}

}  // namespace bq
