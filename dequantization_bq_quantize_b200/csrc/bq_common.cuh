// bq_common.cuh - shared device helpers for the bq kernels (sm_100a).
//
// Element widening, output narrowing, mbarrier / TMA wrappers written as
// inline PTX, and the bounded wait used by every pipelined kernel.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace bq {

// Element type codes, equal to the C ABI's bq_dtype values.
enum : int { kF32 = 0, kF16 = 1, kBF16 = 2 };

template <int DT> struct ElemBytes { static constexpr int value = DT == kF32 ? 4 : 2; };

// Fault word (one per device): bit 0 = a consumer gave up waiting for data,
// bit 1 = a producer gave up waiting for a free stage.
__device__ uint32_t g_fault;

// A wait on an mbarrier gives up after this many nanoseconds (2 s; test
// builds of the fault path set a shorter limit).
#ifndef BQ_WAIT_LIMIT_NS
#define BQ_WAIT_LIMIT_NS 2000000000ull
#endif
constexpr uint64_t kWaitLimitNs = BQ_WAIT_LIMIT_NS;

#ifdef BQ_TEST_HOOKS
// Test builds only (never libbq.so): the producer of the pipelined kernels
// skips the copy of this tile, so that the consumers' wait for it runs out
// and the fault path is exercised without any invalid memory access.
__device__ int64_t g_test_skip_tile = -1;
__device__ __forceinline__ bool test_skip_tile(int64_t tile) { return tile == g_test_skip_tile; }
#else
__device__ __forceinline__ constexpr bool test_skip_tile(int64_t) { return false; }
#endif

// ---------------------------------------------------------------- widening --

// Element j of a 16-bit-element vector held as 32-bit words (element 2i in the
// low half of word i: little-endian order of the bytes in memory).
template <int DT>
__device__ __forceinline__ float widen_pair_elem(uint32_t w, int hi);

template <>
__device__ __forceinline__ float widen_pair_elem<kBF16>(uint32_t w, int hi) {
  return __uint_as_float(hi ? (w & 0xffff0000u) : (w << 16));
}

// fp16 -> fp32 as the mixed-precision add h + (-0.0) (fp16 operand, fp32
// result): exact, with -0 + -0 = -0 and +0 + -0 = +0, and issued on the FMA
// pipe.  The plain conversion measured slower where the kernels widen every
// element (fp16 NF4 blocksize 64 quantize of 1 GiB: 236.0 -> 219.6 us).
template <>
__device__ __forceinline__ float widen_pair_elem<kF16>(uint32_t w, int hi) {
  float d;
  const unsigned short h = static_cast<unsigned short>(hi ? (w >> 16) : (w & 0xffffu));
  asm("add.rn.f32.f16 %0, %1, %2;" : "=f"(d) : "h"(h), "f"(-0.0f));
  return d;
}

// Scalar element load from global memory (any alignment of the element type).
template <int DT>
__device__ __forceinline__ float load_elem(const void* x, int64_t i) {
  if constexpr (DT == kF32) {
    return static_cast<const float*>(x)[i];
  } else {
    uint32_t h = static_cast<const unsigned short*>(x)[i];
    return widen_pair_elem<DT>(h, 0);
  }
}

// --------------------------------------------------------------- narrowing --

// Round-to-nearest-even narrowing of two fp32 values into one 32-bit word
// (first value in the low half).
template <int OT>
__device__ __forceinline__ uint32_t narrow2(float a, float b);

template <>
__device__ __forceinline__ uint32_t narrow2<kBF16>(float a, float b) {
  __nv_bfloat162 v = __floats2bfloat162_rn(a, b);
  return *reinterpret_cast<uint32_t*>(&v);
}

template <>
__device__ __forceinline__ uint32_t narrow2<kF16>(float a, float b) {
  __half2 v = __floats2half2_rn(a, b);
  return *reinterpret_cast<uint32_t*>(&v);
}

template <int OT>
__device__ __forceinline__ void store_elem(void* y, int64_t i, float v) {
  if constexpr (OT == kF32) {
    static_cast<float*>(y)[i] = v;
  } else if constexpr (OT == kBF16) {
    static_cast<__nv_bfloat16*>(y)[i] = __float2bfloat16_rn(v);
  } else {
    static_cast<__half*>(y)[i] = __float2half_rn(v);
  }
}

// ------------------------------------------------ packed fp32 pairs ------

// Two fp32 lanes in one 64-bit register: the sm_100 f32x2 instructions do two
// IEEE operations (round to nearest even, no flush) per instruction.
__device__ __forceinline__ uint64_t pack2(float lo, float hi) {
  uint64_t d;
  asm("mov.b64 %0, {%1, %2};" : "=l"(d) : "f"(lo), "f"(hi));
  return d;
}
__device__ __forceinline__ void unpack2(uint64_t v, float& lo, float& hi) {
  asm("mov.b64 {%0, %1}, %2;" : "=f"(lo), "=f"(hi) : "l"(v));
}
__device__ __forceinline__ uint64_t fma2(uint64_t a, uint64_t b, uint64_t c) {
  uint64_t d;
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(a), "l"(b), "l"(c));
  return d;
}
__device__ __forceinline__ uint64_t mul2(uint64_t a, uint64_t b) {
  uint64_t d;
  asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
  return d;
}

// ----------------------------------------------------- NaN-propagating max --

__device__ __forceinline__ float max_nan(float a, float b) {
  float d;
  asm("max.NaN.f32 %0, %1, %2;" : "=f"(d) : "f"(a), "f"(b));
  return d;
}

__device__ __forceinline__ float min_nan(float a, float b) {
  float d;
  asm("min.NaN.f32 %0, %1, %2;" : "=f"(d) : "f"(a), "f"(b));
  return d;
}

// Packed two-lane signed max / min, NaN-propagating.
template <int DT>
__device__ __forceinline__ uint32_t smax2(uint32_t a, uint32_t b) {
  uint32_t d;
  if constexpr (DT == kBF16) asm("max.NaN.bf16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
  else asm("max.NaN.f16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
  return d;
}
template <int DT>
__device__ __forceinline__ uint32_t smin2(uint32_t a, uint32_t b) {
  uint32_t d;
  if constexpr (DT == kBF16) asm("min.NaN.bf16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
  else asm("min.NaN.f16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
  return d;
}

// Packed two-lane |a| vs |b| max (NaN-propagating) and min; the sign of the
// result is meaningless and dropped later.
template <int DT>
__device__ __forceinline__ uint32_t amax2(uint32_t a, uint32_t b) {
  uint32_t d;
  if constexpr (DT == kBF16) asm("max.NaN.xorsign.abs.bf16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
  else asm("max.NaN.xorsign.abs.f16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
  return d;
}
template <int DT>
__device__ __forceinline__ uint32_t amin2(uint32_t a, uint32_t b) {
  uint32_t d;
  if constexpr (DT == kBF16) asm("min.xorsign.abs.bf16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
  else asm("min.xorsign.abs.f16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
  return d;
}

// ------------------------------------------------------------ PTX wrappers --

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ uint64_t globaltimer_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count)
               : "memory");
}

__device__ __forceinline__ void fence_mbar_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)),
               "r"(bytes)
               : "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}

// Wait until the phase with the given parity has completed; false if that
// does not happen within kWaitLimitNs.
__device__ __forceinline__ bool mbar_wait_bounded(uint64_t* bar, uint32_t parity) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = globaltimer_ns();
  while (true) {
#pragma unroll 1
    for (int i = 0; i < 32; ++i)
      if (mbar_try_wait(bar, parity)) return true;
    if (globaltimer_ns() - t0 > kWaitLimitNs) return false;
  }
}

// 2-D tiled TMA load (no multicast) into this CTA's shared memory, completing
// `bar`'s transaction count.  c0 is the inner (byte) coordinate.
__device__ __forceinline__ void tma_load_2d(void* dst, const CUtensorMap* map, int32_t c0,
                                            int32_t c1, uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%2, %3}], [%4];" ::"r"(smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(c0), "r"(c1), "r"(smem_u32(bar))
      : "memory");
}

// 1-D bulk copy global -> this CTA's shared memory (no multicast); both
// addresses 16-byte aligned and bytes a multiple of 16.  `pol` is an L2
// cache policy (createpolicy).
__device__ __forceinline__ void bulk_load(void* dst, const void* src, uint32_t bytes,
                                          uint64_t* bar, uint64_t pol) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint"
      " [%0], [%1], %2, [%3], %4;"
      ::"r"(smem_u32(dst)), "l"(reinterpret_cast<uint64_t>(src)), "r"(bytes), "r"(smem_u32(bar)),
        "l"(pol)
      : "memory");
}

// For data read once (the codes and scales of a dequantization, GGUF
// blocks): marked evict-first, they leave L2 to the output lines waiting for
// write-back (n = 2^29 NF4 -> bf16, dequantize alone: about 251 -> 244 us).
__device__ __forceinline__ uint64_t l2_evict_first_policy() {
  uint64_t pol;
  asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(pol));
  return pol;
}

// Orders this thread's earlier generic-proxy accesses to shared memory (plain
// loads and stores) before later async-proxy accesses to it (bulk / TMA
// copies).  A consumer that has read a ring stage with plain loads executes it
// before releasing the stage: the producer's next copy into that stage is an
// async-proxy write, which the mbarrier release / acquire alone does not order
// after those loads.
__device__ __forceinline__ void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// Named barrier over `count` threads (a multiple of 32), id != 0.
__device__ __forceinline__ void named_sync(int id, int count) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(count) : "memory");
}

// Named barrier that also returns the OR of `v` over the `count` threads.
__device__ __forceinline__ bool named_sync_or(int id, int count, bool v) {
  uint32_t r;
  asm volatile(
      "{\n\t.reg .pred p, q;\n\t"
      "setp.ne.u32 q, %1, 0;\n\t"
      "bar.red.or.pred p, %2, %3, q;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(r)
      : "r"(static_cast<uint32_t>(v)), "r"(id), "r"(count)
      : "memory");
  return r != 0;
}

__device__ __forceinline__ void record_fault(uint32_t bit) { atomicOr(&g_fault, bit); }

// Programmatic dependent launch.  Kernels are launched so that they may start
// while the previous kernel on the stream is finishing; each one waits for
// that kernel's completion (and its memory) before touching global memory, and
// lets its own dependents start launching right away.
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_release() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

}  // namespace bq
