// bq_probes.cu - test-only CUDA checks of the library's exact arithmetic.
//
// 1. Division: the normalisation the quantize kernels use (per-block
//    reciprocal + Markstein correction, IEEE division for the small-|x| and
//    out-of-range cases) against IEEE division, for every pair of finite
//    bf16 / fp16 values (x, A) with 0 < A and |x| <= A, and for random and
//    edge-heavy fp32 pairs.
// 2. Search: the fast nearest-code search (bucket table or threshold
//    bisection, built on the device from the caller's table) against a plain
//    linear scan of the rule |RN(xn - c_j)| minimal, lowest j on ties, for
//    EVERY float xn in [-1, 1].
// 3. Ordering: a kernel that writes a buffer late while the next kernel on
//    the stream has already started under programmatic dependent launch.
//
// The plain scan here is written independently of the library's code.
#include <cstdint>

#include "bq_search.cuh"

namespace {

__device__ unsigned long long g_mismatch;
__device__ unsigned int g_first_bad_a;
__device__ unsigned int g_first_bad_b;

__device__ __forceinline__ bool same_quotient(float a, float b) {
  // the sign of a zero quotient does not matter to the search
  return __float_as_uint(a) == __float_as_uint(b) || (a == 0.0f && b == 0.0f);
}

// The quantize kernels' bucket path divides elements in pairs for every block
// whose absmax is in [2^-60, 2^60], without a per-element check: with the
// packed Markstein form (div_fast2) for fp32 inputs and the packed two-term
// form (div_fast2_2term) for 16-bit inputs.  It needs the exact quotient,
// except that when the exact quotient is below 2^-38 in magnitude the result
// only has to be below 2^-37.  The safe path uses IEEE division for |x| < A
// 2^-40.  All are checked; the packed forms on both lanes (the second with -x).
__device__ __forceinline__ bool bucket_path_ok(float got, float want) {
  return same_quotient(got, want) || (fabsf(got) < 0x1p-37f && fabsf(want) < 0x1p-38f);
}

template <bool TWO_TERM>
__device__ __forceinline__ bool division_ok(float x, float A) {
  const bq::BlockScale s = bq::make_scale(A);
  const float w0 = __fdiv_rn(x, A), w1 = __fdiv_rn(-x, A);
  bool ok = true;
  if (A >= 0x1p-60f && A <= 0x1p60f) {
    float q0, q1;
    bq::div_fast2(x, -x, s, q0, q1);
    ok = bucket_path_ok(q0, w0) && bucket_path_ok(q1, w1);
    if constexpr (TWO_TERM) {
      bq::div_fast2_2term(x, -x, bq::make_scale_fast_2term(A), q0, q1);
      ok = ok && bucket_path_ok(q0, w0) && bucket_path_ok(q1, w1);
    }
  }
  const float safe = fabsf(x) < s.theta ? bq::div_exact(x, A) : bq::div_fast(x, s);
  return ok && same_quotient(safe, w0);
}

__device__ void report(unsigned int a, unsigned int b) {
  if (atomicAdd(&g_mismatch, 1ull) == 0ull) {
    g_first_bad_a = a;
    g_first_bad_b = b;
  }
}

// 16-bit types: thread handles A = pattern blockIdx-derived, x over all.
template <int DT>
__global__ void div16_all(int a_lo) {
  const uint32_t a_bits = static_cast<uint32_t>(a_lo) + blockIdx.x;
  const float A = bq::widen_pair_elem<DT>(a_bits, 0);
  if (!(A > 0.0f) || !isfinite(A)) return;
  for (uint32_t xb = threadIdx.x; xb < 65536u; xb += blockDim.x) {
    const float x = bq::widen_pair_elem<DT>(xb, 0);
    if (!isfinite(x) || !(fabsf(x) <= A)) continue;
    if (!division_ok<true>(x, A)) report(xb, a_bits);
  }
}

__device__ __forceinline__ uint32_t mix(uint64_t v) {
  v ^= v >> 33; v *= 0xff51afd7ed558ccdull;
  v ^= v >> 33; v *= 0xc4ceb9fe1a85ec53ull;
  v ^= v >> 33;
  return static_cast<uint32_t>(v);
}

__global__ void div32_random(uint64_t count, uint64_t seed) {
  const uint64_t stride = static_cast<uint64_t>(gridDim.x) * blockDim.x;
  for (uint64_t i = blockIdx.x * static_cast<uint64_t>(blockDim.x) + threadIdx.x; i < count;
       i += stride) {
    uint32_t ab = mix(seed + 2 * i), xb = mix(seed + 2 * i + 1);
    const uint32_t kind = i & 3;
    if (kind == 1) ab |= 0x007fffffu;            // all-ones mantissa
    if (kind == 2) xb |= 0x007fffffu;
    if (kind == 3) ab = (ab & 0xff800000u) | 0x00000001u;
    ab &= 0x7fffffffu;
    float A = __uint_as_float(ab);
    float x = __uint_as_float(xb);
    if (!isfinite(A) || !isfinite(x) || A == 0.0f) continue;
    if (fabsf(x) > A) { const float t = A; A = fabsf(x); x = copysignf(t, x); }
    if (!division_ok<false>(x, A)) report(__float_as_uint(x), __float_as_uint(A));
  }
}

// ------------------------------------------------------------- search ----

template <int E>
struct ProbeSmem {
  bq::TableSmem tab;
  bq::Lut<E> lut;
  float c[E];
};

template <int E>
__device__ uint32_t plain_scan(float xn, const float* c) {
  uint32_t best_j = 0;
  float best = fabsf(__fsub_rn(xn, c[0]));
  for (int j = 1; j < E; ++j) {
    const float d = fabsf(__fsub_rn(xn, c[j]));
    if (d < best) { best = d; best_j = j; }
  }
  return best_j;
}

// Every float in [-1, 1]: positive bit patterns 0..0x3f800000 and their negatives.
template <int E>
__global__ void __launch_bounds__(256) search_all(const float* code, int* mode_out) {
  extern __shared__ uint8_t raw[];
  ProbeSmem<E>& s = *reinterpret_cast<ProbeSmem<E>*>(raw);
  const int ct = threadIdx.x;
  bq::build_search<E, 256>(s.tab, s.lut, code, ct);
  if (ct < E) s.c[ct] = code[ct];
  __syncthreads();
  const int mode = s.tab.mode;
  if (blockIdx.x == 0 && ct == 0) *mode_out = mode;
  const uint64_t npos = 0x3f800001ull;
  const uint64_t total = 2 * npos;
  const uint64_t stride = static_cast<uint64_t>(gridDim.x) * blockDim.x;
  for (uint64_t i = blockIdx.x * static_cast<uint64_t>(blockDim.x) + ct; i < total; i += stride) {
    const uint32_t bits = i < npos ? static_cast<uint32_t>(i)
                                   : (static_cast<uint32_t>(i - npos) | 0x80000000u);
    const float xn = __uint_as_float(bits);
    uint32_t got;
    if (mode == bq::kModeLutF) got = bq::search<E, bq::kModeLutF>(xn, s.tab, s.lut);
    else if (mode == bq::kModeLutI)
      got = bq::search<E, E == 256 ? bq::kModeLutI : bq::kModeLutF>(xn, s.tab, s.lut);
    else if (mode == bq::kModeLut) got = bq::search<E, bq::kModeLut>(xn, s.tab, s.lut);
    else if (mode == bq::kModeBsearch) got = bq::search<E, bq::kModeBsearch>(xn, s.tab, s.lut);
    else got = bq::search<E, bq::kModeScan>(xn, s.tab, s.lut);
    const uint32_t want = plain_scan<E>(xn, s.c);
    if (got != want) report(bits, (got << 16) | want);
  }
}

template <int E, int MODE>
__global__ void __launch_bounds__(256) search_forced(const float* code, int* mode_out) {
  // same sweep, but with a forced search form: the bisection form (built for
  // every valid table), or the float-select form of a 256-entry table that
  // would otherwise get the integer form (built with that form disallowed)
  extern __shared__ uint8_t raw[];
  ProbeSmem<E>& s = *reinterpret_cast<ProbeSmem<E>*>(raw);
  const int ct = threadIdx.x;
  bq::build_search<E, 256>(s.tab, s.lut, code, ct, MODE != bq::kModeLutF);
  if (ct < E) s.c[ct] = code[ct];
  __syncthreads();
  if (blockIdx.x == 0 && ct == 0) *mode_out = s.tab.mode;
  if (s.tab.mode == bq::kModeScan) return;   // forced forms need a valid table
  if (MODE == bq::kModeLutF && s.tab.mode != bq::kModeLutF) return;  // reported via mode_out
  const uint64_t npos = 0x3f800001ull;
  const uint64_t total = 2 * npos;
  const uint64_t stride = static_cast<uint64_t>(gridDim.x) * blockDim.x;
  for (uint64_t i = blockIdx.x * static_cast<uint64_t>(blockDim.x) + ct; i < total; i += stride) {
    const uint32_t bits = i < npos ? static_cast<uint32_t>(i)
                                   : (static_cast<uint32_t>(i - npos) | 0x80000000u);
    const float xn = __uint_as_float(bits);
    const uint32_t got = bq::search<E, MODE>(xn, s.tab, s.lut);
    const uint32_t want = plain_scan<E>(xn, s.c);
    if (got != want) report(bits, (got << 16) | want);
  }
}

// ------------------------------------------------------- bounded wait ----

// One thread waits on an mbarrier that nothing ever arrives on.  The wait must
// give up by itself (bounded by bq::kWaitLimitNs) and report it; the context
// stays usable afterwards.
__global__ void wait_timeout(int* result) {
  __shared__ uint64_t bar;
  if (threadIdx.x == 0) {
    bq::mbar_init(&bar, 1);
    bq::fence_mbar_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    const uint64_t t0 = bq::globaltimer_ns();
    const bool ok = bq::mbar_wait_bounded(&bar, 0);
    const uint64_t t1 = bq::globaltimer_ns();
    result[0] = ok ? 1 : 0;
    result[1] = static_cast<int>((t1 - t0) / 1000000ull);
  }
}

// ------------------------------------------------ late writer (PDL) ----

// Launched with programmatic stream serialization: waits for the work before
// it, lets the next kernel on the stream start launching at once, spins for
// spin_ns (ended by the timer), then copies count floats from src to dst.  A
// kernel launched after it the same way runs the part before its own
// dependent-launch wait while dst still holds the old values.
// The stores are volatile asm: the timer reads of the spin touch no memory,
// so plain stores could legally be performed before the spin.
__global__ void late_writer(float* dst, const float* src, int count, uint64_t spin_ns) {
  bq::pdl_wait();
  bq::pdl_release();
  const uint64_t t0 = bq::globaltimer_ns();
  while (bq::globaltimer_ns() - t0 < spin_ns) {
  }
  for (int i = threadIdx.x; i < count; i += blockDim.x) {
    const float v = src[i];
    asm volatile("st.global.f32 [%0], %1;" ::"l"(dst + i), "f"(v) : "memory");
  }
}

// Reads p[idx] at L2 before and after its dependent-launch wait.  The first
// value is put in shared memory behind a barrier before the wait, as the
// quantize kernel does with the codebook it builds its tables from: a load
// whose value is only used after the wait may be performed after it.
__global__ void early_reader(const float* p, int idx, float* out) {
  __shared__ float before;
  if (threadIdx.x == 0) before = __ldcg(p + idx);
  __syncthreads();
  bq::pdl_wait();
  if (threadIdx.x == 0) {
    out[0] = before;
    out[1] = __ldcg(p + idx);
  }
}

// Timestamps (globaltimer, ns) of a late_writer-like kernel and of the kernel
// launched after it: t[0] writer start, t[1] writer end of spin, t[2] reader
// start, t[3] reader after its wait.
__global__ void timed_writer(unsigned long long* t, uint64_t spin_ns) {
  bq::pdl_wait();
  bq::pdl_release();
  const uint64_t t0 = bq::globaltimer_ns();
  while (bq::globaltimer_ns() - t0 < spin_ns) {
  }
  if (threadIdx.x == 0) {
    t[0] = t0;
    t[1] = bq::globaltimer_ns();
  }
}
// late_writer and early_reader with timestamps: t[0] writer start, t[1]
// writer just before its store, t[2] reader start, t[3] reader after its
// first load reached shared memory, t[4] reader after its wait; t[5], t[6]
// the bits of the values read before and after the wait.
__global__ void timed_late_writer(float* dst, const float* src, unsigned long long* t,
                                  uint64_t spin_ns) {
  bq::pdl_wait();
  bq::pdl_release();
  const uint64_t t0 = bq::globaltimer_ns();
  while (bq::globaltimer_ns() - t0 < spin_ns) {
  }
  const uint64_t t1 = bq::globaltimer_ns();
  if (threadIdx.x == 0) {
    const float v = src[1];
    asm volatile("st.global.f32 [%0], %1;" ::"l"(dst + 1), "f"(v) : "memory");
    t[0] = t0;
    t[1] = t1;
  }
}
__global__ void timed_early_reader(const float* p, unsigned long long* t) {
  __shared__ float before;
  const uint64_t t2 = bq::globaltimer_ns();
  if (threadIdx.x == 0) before = __ldcg(p + 1);
  __syncthreads();
  const uint64_t t3 = bq::globaltimer_ns();
  bq::pdl_wait();
  const uint64_t t4 = bq::globaltimer_ns();
  if (threadIdx.x == 0) {
    t[2] = t2;
    t[3] = t3;
    t[4] = t4;
    t[5] = __float_as_uint(before);
    t[6] = __float_as_uint(__ldcg(p + 1));
  }
}
__global__ void timed_reader(unsigned long long* t) {
  const uint64_t t2 = bq::globaltimer_ns();
  bq::pdl_wait();
  if (threadIdx.x == 0) {
    t[2] = t2;
    t[3] = bq::globaltimer_ns();
  }
}

template <typename... KArgs, typename... Args>
cudaError_t launch_pdl1(void (*kernel)(KArgs...), cudaStream_t stream, Args... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(1);
  cfg.blockDim = dim3(32);
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kernel, args...);
}

int g_sms = 0;

cudaError_t reset() {
  unsigned long long z = 0;
  unsigned int zi = 0;
  cudaError_t e = cudaMemcpyToSymbol(g_mismatch, &z, sizeof(z));
  if (e == cudaSuccess) e = cudaMemcpyToSymbol(g_first_bad_a, &zi, sizeof(zi));
  if (e == cudaSuccess) e = cudaMemcpyToSymbol(g_first_bad_b, &zi, sizeof(zi));
  if (e == cudaSuccess && g_sms == 0) {
    int dev = 0;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&g_sms, cudaDevAttrMultiProcessorCount, dev);
  }
  return e;
}

int finish(unsigned long long* mismatches, unsigned int* first_a, unsigned int* first_b) {
  cudaError_t e = cudaGetLastError();
  if (e == cudaSuccess) e = cudaDeviceSynchronize();
  if (e == cudaSuccess) e = cudaMemcpyFromSymbol(mismatches, g_mismatch, sizeof(*mismatches));
  if (e == cudaSuccess) e = cudaMemcpyFromSymbol(first_a, g_first_bad_a, sizeof(*first_a));
  if (e == cudaSuccess) e = cudaMemcpyFromSymbol(first_b, g_first_bad_b, sizeof(*first_b));
  return static_cast<int>(e);
}

// mode_out is a HOST pointer: the kernel writes the chosen search form into a
// device word, copied back after the sweep.
template <int E, typename K>
int run_search(K kernel, const float* code, int* mode_out, unsigned long long* mm,
               unsigned int* fa, unsigned int* fb) {
  cudaError_t e = reset();
  if (e != cudaSuccess) return static_cast<int>(e);
  const size_t smem = sizeof(ProbeSmem<E>);
  e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
  if (e != cudaSuccess) return static_cast<int>(e);
  int* d_mode = nullptr;
  e = cudaMalloc(&d_mode, sizeof(int));
  if (e != cudaSuccess) return static_cast<int>(e);
  kernel<<<g_sms * 4, 256, smem>>>(code, d_mode);
  int rc = finish(mm, fa, fb);
  if (rc == 0) rc = static_cast<int>(cudaMemcpy(mode_out, d_mode, sizeof(int), cudaMemcpyDeviceToHost));
  cudaFree(d_mode);
  return rc;
}

}  // namespace

extern "C" {

// dtype: 1 = fp16, 2 = bf16.  Returns a cudaError_t value.
__attribute__((visibility("default"))) int probe_div16(int dtype, unsigned long long* mm,
                                                       unsigned int* fa, unsigned int* fb) {
  cudaError_t e = reset();
  if (e != cudaSuccess) return static_cast<int>(e);
  // A over all positive patterns 0x0001..0x7fff (65535 CTAs)
  if (dtype == 1) div16_all<bq::kF16><<<0x7fff, 256>>>(1);
  else div16_all<bq::kBF16><<<0x7fff, 256>>>(1);
  return finish(mm, fa, fb);
}

__attribute__((visibility("default"))) int probe_div32(unsigned long long count,
                                                       unsigned long long seed,
                                                       unsigned long long* mm, unsigned int* fa,
                                                       unsigned int* fb) {
  cudaError_t e = reset();
  if (e != cudaSuccess) return static_cast<int>(e);
  div32_random<<<g_sms * 8, 256>>>(count, seed);
  return finish(mm, fa, fb);
}

// mode_request: -1 = whatever the builder picks, 1 = force the bisection form,
// 3 = the float-select form of a 256-entry table (integer form disallowed).
__attribute__((visibility("default"))) int probe_search(const float* code, int entries,
                                                        int mode_request, int* mode_out,
                                                        unsigned long long* mm, unsigned int* fa,
                                                        unsigned int* fb) {
  if (entries == 16) {
    if (mode_request == 1)
      return run_search<16>(search_forced<16, bq::kModeBsearch>, code, mode_out, mm, fa, fb);
    return run_search<16>(search_all<16>, code, mode_out, mm, fa, fb);
  }
  if (mode_request == 1)
    return run_search<256>(search_forced<256, bq::kModeBsearch>, code, mode_out, mm, fa, fb);
  if (mode_request == 3)
    return run_search<256>(search_forced<256, bq::kModeLutF>, code, mode_out, mm, fa, fb);
  return run_search<256>(search_all<256>, code, mode_out, mm, fa, fb);
}

// result[0] = 1 if the wait completed (it must not), result[1] = ms waited.
// Enqueue late_writer on `stream` (spin at most 0.2 s, at most 4096 floats).
__attribute__((visibility("default"))) int probe_late_write(float* dst, const float* src,
                                                            int count,
                                                            unsigned long long spin_ns,
                                                            cudaStream_t stream) {
  if (count < 0 || count > 4096 || spin_ns > 200000000ull) return cudaErrorInvalidValue;
  return static_cast<int>(launch_pdl1(late_writer, stream, dst, src, count,
                                      static_cast<uint64_t>(spin_ns)));
}

// Enqueue early_reader on `stream`: out[0] = p[idx] before its wait, out[1]
// after (both device pointers).
__attribute__((visibility("default"))) int probe_early_read(const float* p, int idx, float* out,
                                                            cudaStream_t stream) {
  return static_cast<int>(launch_pdl1(early_reader, stream, p, idx, out));
}

// The two timed kernels back to back on `stream`; t: 4 device words.
__attribute__((visibility("default"))) int probe_pdl_timing(unsigned long long* t,
                                                            unsigned long long spin_ns,
                                                            cudaStream_t stream) {
  if (spin_ns > 200000000ull) return cudaErrorInvalidValue;
  cudaError_t e = launch_pdl1(timed_writer, stream, t, static_cast<uint64_t>(spin_ns));
  if (e == cudaSuccess) e = launch_pdl1(timed_reader, stream, t);
  return static_cast<int>(e);
}

// timed_late_writer then timed_early_reader on `stream`; t: 7 device words.
__attribute__((visibility("default"))) int probe_pdl_timing2(float* dst, const float* src,
                                                             unsigned long long* t,
                                                             unsigned long long spin_ns,
                                                             cudaStream_t stream) {
  if (spin_ns > 200000000ull) return cudaErrorInvalidValue;
  cudaError_t e = launch_pdl1(timed_late_writer, stream, dst, src, t,
                              static_cast<uint64_t>(spin_ns));
  if (e == cudaSuccess) e = launch_pdl1(timed_early_reader, stream, static_cast<const float*>(dst), t);
  return static_cast<int>(e);
}

__attribute__((visibility("default"))) int probe_wait_timeout(int* result) {
  int* d = nullptr;
  cudaError_t e = cudaMalloc(&d, 2 * sizeof(int));
  if (e != cudaSuccess) return static_cast<int>(e);
  wait_timeout<<<1, 32>>>(d);
  e = cudaGetLastError();
  if (e == cudaSuccess) e = cudaDeviceSynchronize();
  if (e == cudaSuccess) e = cudaMemcpy(result, d, 2 * sizeof(int), cudaMemcpyDeviceToHost);
  cudaFree(d);
  return static_cast<int>(e);
}

}  // extern "C"
