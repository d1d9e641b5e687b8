// bq_api.cu - the C ABI of libbq.so (declared in include/bq.h): host-side
// validation, launch-configuration choice, TMA descriptor encoding, error
// reporting.  All kernels live in this one translation unit.
#include "bq.h"

#include <cudaTypedefs.h>

#include <atomic>
#include <cstdio>
#include <cstring>
#include <mutex>
#include <string>
#include <utility>

#include "bq_dequant.cuh"
#include "bq_dequant_stream.cuh"
#include "bq_gguf.cuh"
#include "bq_gguf_encode.cuh"
#include "bq_quantize.cuh"

static_assert(int(BQ_F32) == int(bq::kF32) && int(BQ_F16) == int(bq::kF16) &&
                  int(BQ_BF16) == int(bq::kBF16),
              "dtype codes must match");

namespace {

thread_local std::string t_err;

bq_status cuda_fail(cudaError_t e, const char* what) {
  t_err = std::string(what) + ": " + cudaGetErrorString(e);
  return BQ_ERR_CUDA;
}

constexpr int kMaxDevices = 64;

// Per-device facts, read once per device.
struct DevInfo {
  int sms = 0;
};
DevInfo g_dev[kMaxDevices];
std::once_flag g_dev_once[kMaxDevices];

bq_status current_device(int* dev, DevInfo* info) {
  cudaError_t e = cudaGetDevice(dev);
  if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
  if (*dev < 0 || *dev >= kMaxDevices) {
    t_err = "device ordinal out of range";
    return BQ_ERR_UNSUPPORTED;
  }
  cudaError_t ie = cudaSuccess;
  std::call_once(g_dev_once[*dev], [&] {
    ie = cudaDeviceGetAttribute(&g_dev[*dev].sms, cudaDevAttrMultiProcessorCount, *dev);
  });
  if (ie != cudaSuccess) return cuda_fail(ie, "cudaDeviceGetAttribute");
  if (g_dev[*dev].sms <= 0) {
    t_err = "device attributes unavailable";
    return BQ_ERR_CUDA;
  }
  *info = g_dev[*dev];
  return BQ_OK;
}

// Per (kernel, device) one-time set-up: dynamic shared memory limit and the
// number of resident CTAs per SM.
struct KernelSlot {
  std::once_flag once[kMaxDevices];
  int occ[kMaxDevices] = {};
  cudaError_t err[kMaxDevices] = {};
};

template <typename K>
bq_status kernel_occupancy(KernelSlot& slot, K kernel, int dev, int threads, size_t smem,
                           int* occ) {
  std::call_once(slot.once[dev], [&] {
    cudaError_t e = cudaSuccess;
    if (smem > 48 * 1024)
      e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               static_cast<int>(smem));
    int o = 0;
    if (e == cudaSuccess) e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&o, kernel, threads, smem);
    slot.err[dev] = e;
    slot.occ[dev] = o;
  });
  if (slot.err[dev] != cudaSuccess) return cuda_fail(slot.err[dev], "kernel set-up");
  *occ = slot.occ[dev] > 0 ? slot.occ[dev] : 1;
  return BQ_OK;
}

// cuTensorMapEncodeTiled from the driver, fetched through the runtime.
PFN_cuTensorMapEncodeTiled_v12000 encode_tiled() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &p, 12000, cudaEnableDefault,
                                         &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  });
  return fn;
}

// Launch with programmatic stream serialization: the kernel may begin while
// the previous kernel on the stream finishes; every kernel waits for it
// (griddepcontrol.wait) before touching global memory.
template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*kernel)(KArgs...), int grid, int block, size_t smem,
                       cudaStream_t stream, Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(grid));
  cfg.blockDim = dim3(static_cast<unsigned>(block));
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
}

bool valid_dtype(int d) { return d == BQ_F32 || d == BQ_F16 || d == BQ_BF16; }
int elem_bytes(int d) { return d == BQ_F32 ? 4 : 2; }
bool valid_blocksize(int32_t bs) { return bs >= 32 && bs <= 4096 && (bs & (bs - 1)) == 0; }
int log2i(int32_t v) { int l = 0; while ((1 << l) < v) ++l; return l; }
bool aligned(const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) & (a - 1)) == 0; }

// ------------------------------------------------------------- quantize ---

template <int DT, int E, int TPB>
bq_status launch_quantize(const bq::QParams& p, const CUtensorMap& map, int dev, int sms,
                          cudaStream_t stream) {
  static KernelSlot slot;
  auto kernel = bq::quantize_kernel<DT, E, TPB>;
  constexpr size_t smem = bq::qsmem_bytes<E>();
  int occ = 1;
  constexpr int threads = bq::q_threads<DT, E, TPB>();
  bq_status s = kernel_occupancy(slot, kernel, dev, threads, smem, &occ);
  if (s != BQ_OK) return s;
  constexpr int BPT = bq::kQConsumers / TPB;
  const int64_t gen_blocks = p.nb - p.full_tiles * BPT;
  int64_t want = p.full_tiles;
  const int64_t want_gen = (gen_blocks + bq::kQConsumerWarps - 1) / bq::kQConsumerWarps;
  if (want_gen > want) want = want_gen;
  if (want < 1) want = 1;
  const int64_t cap = static_cast<int64_t>(occ) * sms;
  const int grid = static_cast<int>(want < cap ? want : cap);
  cudaError_t e = launch_pdl(kernel, grid, threads, smem, stream, map, p);
  return e == cudaSuccess ? BQ_OK : cuda_fail(e, "quantize launch");
}

template <int DT, int E>
bq_status dispatch_quantize_bs(const bq::QParams& p, const CUtensorMap& map, int dev, int sms,
                               cudaStream_t stream) {
  // threads per quantization block: each consumer thread owns 64 bytes
  constexpr int EPT = bq::kThreadBytes / bq::ElemBytes<DT>::value;
  switch (p.bs / EPT) {
    case 1: if constexpr (EPT == 32) return launch_quantize<DT, E, 1>(p, map, dev, sms, stream); break;
    case 2: return launch_quantize<DT, E, 2>(p, map, dev, sms, stream);
    case 4: return launch_quantize<DT, E, 4>(p, map, dev, sms, stream);
    case 8: return launch_quantize<DT, E, 8>(p, map, dev, sms, stream);
    case 16: return launch_quantize<DT, E, 16>(p, map, dev, sms, stream);
    case 32: return launch_quantize<DT, E, 32>(p, map, dev, sms, stream);
    case 64: return launch_quantize<DT, E, 64>(p, map, dev, sms, stream);
    case 128: return launch_quantize<DT, E, 128>(p, map, dev, sms, stream);
    case 256: if constexpr (EPT == 16) return launch_quantize<DT, E, 256>(p, map, dev, sms, stream); break;
    default: break;
  }
  t_err = "no kernel for this blocksize";
  return BQ_ERR_UNSUPPORTED;
}

template <int DT>
bq_status dispatch_quantize(const bq::QParams& p, int entries, const CUtensorMap& map, int dev,
                            int sms, cudaStream_t stream) {
  if (entries == 16) return dispatch_quantize_bs<DT, 16>(p, map, dev, sms, stream);
  return dispatch_quantize_bs<DT, 256>(p, map, dev, sms, stream);
}

// ----------------------------------------------------------- dequantize ---

template <int E, int OT, bool NESTED>
bq_status launch_dequant(const bq::DParams& p, int dev, int sms, cudaStream_t stream) {
  static KernelSlot slot;
  auto kernel = bq::dequant_kernel<E, OT, NESTED>;
  int occ = 1;
  bq_status s = kernel_occupancy(slot, kernel, dev, bq::kDThreads, 0, &occ);
  if (s != BQ_OK) return s;
  const int64_t work = p.vec ? (p.nchunks + 3) / 4 + 1 : p.n;
  int64_t want = (work + bq::kDThreads - 1) / bq::kDThreads;
  // up to four waves of resident CTAs: the stores of more CTAs spread over
  // more of the output at once (8-bit codes: 297 -> 284 us at n = 2^29
  // bf16; 4-bit codes unchanged)
  const int64_t cap = static_cast<int64_t>(occ) * sms * 4;
  if (want > cap) want = cap;
  if (want < 1) want = 1;
  cudaError_t e = launch_pdl(kernel, static_cast<int>(want), bq::kDThreads, 0, stream, p);
  return e == cudaSuccess ? BQ_OK : cuda_fail(e, "dequantize launch");
}

template <int OT, bool NESTED>
bq_status dispatch_dequant(const bq::DParams& p, int entries, int dev, int sms, cudaStream_t st) {
  if (entries == 16) return launch_dequant<16, OT, NESTED>(p, dev, sms, st);
  return launch_dequant<256, OT, NESTED>(p, dev, sms, st);
}

template <int E, int OT, bool NESTED, bool ADIRECT = false>
bq_status launch_dequant_stream(const bq::DParams& p, int64_t ntiles, int dev, int sms,
                                cudaStream_t stream) {
  static KernelSlot slot;
  auto kernel = bq::dequant_stream_kernel<E, OT, NESTED, ADIRECT>;
  constexpr size_t smem = bq::ssmem_bytes<E>();
  int occ = 1;
  bq_status s = kernel_occupancy(slot, kernel, dev, bq::kSThreads, smem, &occ);
  if (s != BQ_OK) return s;
  int64_t want = static_cast<int64_t>(occ) * sms;
  if (want > ntiles) want = ntiles;
  if (want < 1) want = 1;
  cudaError_t e = launch_pdl(kernel, static_cast<int>(want), bq::kSThreads, smem, stream, p, ntiles);
  return e == cudaSuccess ? BQ_OK : cuda_fail(e, "dequantize launch");
}

// Shared by the plain and the compressed-statistics dequantization: p.q,
// p.absmax or (p.qa, p.absmax2, p.code2, p.bs2_log2), p.code and p.y are set
// and validated by the caller.
template <bool NESTED>
bq_status dequant_entry(bq::DParams p, int64_t n, int32_t blocksize, int32_t code_entries,
                        bq_dtype y_dtype, cudaStream_t stream) {
  int dev;
  DevInfo info;
  bq_status s = current_device(&dev, &info);
  if (s != BQ_OK) return s;
  p.n = n;
  p.bs_log2 = log2i(blocksize);
  const int ce = 16 / elem_bytes(y_dtype);
  const int qb = code_entries == 16 ? ce / 2 : ce;
  p.vec = aligned(p.y, 16) && aligned(p.q, qb);
  p.nchunks = p.vec ? n / ce : 0;
  // 4-bit codes, 16-byte aligned buffers, 16-bit outputs, at least one whole
  // tile, and a tile's statistics slice a whole number of 16-byte units
  // (plain: 4-byte scales, blocksize <= 2048; nested: 1-byte codes,
  // blocksize <= 512, and one second-level scale per tile), or plain
  // blocksize 4096 (the producer copies the tile's two scales): stream the
  // codes through shared memory.  (8-bit codes measured faster on
  // dequant_kernel: their 8 KiB stages and 32-copy table leave 3 CTAs per
  // SM.  So did fp32 outputs, whose stores are twice as many per code byte:
  // 1 GiB fp32 NF4, 207-211 us against 214-222 us streamed.)
  const bool stream_ok =
      NESTED ? (aligned(p.qa, 16) && blocksize <= 512 &&
                int64_t{blocksize} << p.bs2_log2 >= bq::kSTile)
             : (aligned(p.absmax, 16) || blocksize > 2048);
  if (stream_ok && code_entries == 16 && aligned(p.y, 16) && aligned(p.q, 16) &&
      y_dtype != BQ_F32 && n >= bq::kSTile) {
    const int64_t ntiles = n / bq::kSTile;
    if constexpr (!NESTED) {
      if (blocksize > 2048) {
        if (y_dtype == BQ_F16)
          return launch_dequant_stream<16, bq::kF16, false, true>(p, ntiles, dev, info.sms, stream);
        return launch_dequant_stream<16, bq::kBF16, false, true>(p, ntiles, dev, info.sms, stream);
      }
    }
    if (y_dtype == BQ_F16)
      return launch_dequant_stream<16, bq::kF16, NESTED>(p, ntiles, dev, info.sms, stream);
    return launch_dequant_stream<16, bq::kBF16, NESTED>(p, ntiles, dev, info.sms, stream);
  }
  switch (y_dtype) {
    case BQ_F32: return dispatch_dequant<bq::kF32, NESTED>(p, code_entries, dev, info.sms, stream);
    case BQ_F16: return dispatch_dequant<bq::kF16, NESTED>(p, code_entries, dev, info.sms, stream);
    default: return dispatch_dequant<bq::kBF16, NESTED>(p, code_entries, dev, info.sms, stream);
  }
}

// ----------------------------------------------------------------- GGUF ---

template <int KIND, int OT>
bq_status launch_gguf(const bq::GParams& p, int dev, int sms, cudaStream_t stream) {
  static KernelSlot slot;
  auto kernel = bq::gguf_kernel<KIND, OT>;
  int occ = 1;
  bq_status s = kernel_occupancy(slot, kernel, dev, bq::kGThreads, 0, &occ);
  if (s != BQ_OK) return s;
  constexpr int kStep = bq::GStep<KIND>::value;
  const int64_t steps = (p.n_blocks + kStep - 1) / kStep;
  int64_t want = (steps + bq::kGThreads / 32 - 1) / (bq::kGThreads / 32);
  // up to four waves of resident CTAs (Q4_K 4096 x 14336: 31.8 -> 28.7 us)
  const int64_t cap = static_cast<int64_t>(occ) * sms * 4;
  if (want > cap) want = cap;
  if (want < 1) want = 1;
  cudaError_t e = launch_pdl(kernel, static_cast<int>(want), bq::kGThreads, 0, stream, p);
  return e == cudaSuccess ? BQ_OK : cuda_fail(e, "gguf dequant launch");
}

template <int KIND>
bq_status gguf_entry(const void* blocks, int64_t n_blocks, void* y, bq_dtype y_dtype,
                     cudaStream_t stream) {
  t_err.clear();
  if (n_blocks < 0 || !valid_dtype(y_dtype)) return BQ_ERR_INVALID_ARG;
  if (n_blocks == 0) return BQ_OK;
  if (n_blocks > (int64_t{1} << 52)) return BQ_ERR_INVALID_ARG;
  if (!blocks || !y || !aligned(y, elem_bytes(y_dtype))) return BQ_ERR_INVALID_ARG;
  int dev;
  DevInfo info;
  bq_status s = current_device(&dev, &info);
  if (s != BQ_OK) return s;
  bq::GParams p;
  p.blocks = static_cast<const uint8_t*>(blocks);
  p.y = y;
  p.n_blocks = n_blocks;
  p.vec = aligned(blocks, 16) && aligned(y, 16);
  switch (y_dtype) {
    case BQ_F32: return launch_gguf<KIND, bq::kF32>(p, dev, info.sms, stream);
    case BQ_F16: return launch_gguf<KIND, bq::kF16>(p, dev, info.sms, stream);
    default: return launch_gguf<KIND, bq::kBF16>(p, dev, info.sms, stream);
  }
}

template <int OT>
bq_status launch_bf16(const bq::BParams& p, int dev, int sms, cudaStream_t stream) {
  static KernelSlot slot;
  auto kernel = bq::bf16_kernel<OT>;
  int occ = 1;
  bq_status s = kernel_occupancy(slot, kernel, dev, bq::kGThreads, 0, &occ);
  if (s != BQ_OK) return s;
  const int64_t work = p.ngroups > 0 ? p.ngroups : p.n;
  int64_t want = (work + bq::kGThreads - 1) / bq::kGThreads;
  const int64_t cap = static_cast<int64_t>(occ) * sms;
  if (want > cap) want = cap;
  if (want < 1) want = 1;
  cudaError_t e = launch_pdl(kernel, static_cast<int>(want), bq::kGThreads, 0, stream, p);
  return e == cudaSuccess ? BQ_OK : cuda_fail(e, "bf16 conversion launch");
}

template <int KIND, int IT>
bq_status launch_gguf_encode(const bq::GEParams& p, int dev, int sms, cudaStream_t stream) {
  static KernelSlot slot;
  auto kernel = bq::gguf_encode_kernel<KIND, IT>;
  int occ = 1;
  bq_status s = kernel_occupancy(slot, kernel, dev, bq::kGThreads, 0, &occ);
  if (s != BQ_OK) return s;
  const int64_t steps = (p.n_blocks + 31) / 32;
  int64_t want = (steps + bq::kGThreads / 32 - 1) / (bq::kGThreads / 32);
  // one wave of resident CTAs (four waves measured slower for the encoders)
  const int64_t cap = static_cast<int64_t>(occ) * sms;
  if (want > cap) want = cap;
  if (want < 1) want = 1;
  cudaError_t e = launch_pdl(kernel, static_cast<int>(want), bq::kGThreads, 0, stream, p);
  return e == cudaSuccess ? BQ_OK : cuda_fail(e, "gguf encode launch");
}

template <int KIND>
bq_status gguf_encode_entry(const void* x, bq_dtype x_dtype, int64_t n, void* blocks,
                            cudaStream_t stream) {
  t_err.clear();
  if (n < 0 || n % 32 != 0 || !valid_dtype(x_dtype)) return BQ_ERR_INVALID_ARG;
  if (n == 0) return BQ_OK;
  if (n > (int64_t{1} << 50)) return BQ_ERR_INVALID_ARG;
  if (!x || !blocks || !aligned(x, elem_bytes(x_dtype))) return BQ_ERR_INVALID_ARG;
  int dev;
  DevInfo info;
  bq_status s = current_device(&dev, &info);
  if (s != BQ_OK) return s;
  bq::GEParams p;
  p.x = x;
  p.blocks = static_cast<uint8_t*>(blocks);
  p.n_blocks = n / 32;
  p.vec = aligned(x, 16) && aligned(blocks, 16);
  switch (x_dtype) {
    case BQ_F32: return launch_gguf_encode<KIND, bq::kF32>(p, dev, info.sms, stream);
    case BQ_F16: return launch_gguf_encode<KIND, bq::kF16>(p, dev, info.sms, stream);
    default: return launch_gguf_encode<KIND, bq::kBF16>(p, dev, info.sms, stream);
  }
}

}  // namespace

// ------------------------------------------ allocation-free nested quantize ---

// First-level fp32 statistics of bq_quantize_blockwise_nested_noalloc: one
// array per device, held from the library's load on that device until the
// process exits, shared by every call (see include/bq.h).  Host code must not
// pass this name to a kernel: on the host it is a stand-in object, not the
// device address, which noalloc_stats() looks up.
static __device__ __align__(256) float g_noalloc_stats[BQ_NOALLOC_MAX_BLOCKS];

namespace {

std::once_flag g_noalloc_once[kMaxDevices];
float* g_noalloc_ptr[kMaxDevices] = {};
cudaError_t g_noalloc_err[kMaxDevices] = {};

// Device address of g_noalloc_stats on `dev`, looked up once per device with
// that device current (the caller's current device).
bq_status noalloc_stats(int dev, float** ptr) {
  std::call_once(g_noalloc_once[dev], [&] {
    void* p = nullptr;
    g_noalloc_err[dev] = cudaGetSymbolAddress(&p, g_noalloc_stats);
    g_noalloc_ptr[dev] = static_cast<float*>(p);
  });
  if (g_noalloc_err[dev] != cudaSuccess)
    return cuda_fail(g_noalloc_err[dev], "looking up the static statistics array");
  if (!g_noalloc_ptr[dev]) {
    t_err = "static statistics array has no device address";
    return BQ_ERR_CUDA;
  }
  *ptr = g_noalloc_ptr[dev];
  return BQ_OK;
}

}  // namespace

// ===================================================================== ABI ==

extern "C" {

bq_status bq_quantize_blockwise(const void* x, bq_dtype x_dtype, int64_t n, int32_t blocksize,
                                const float* code, int32_t code_entries, float* absmax,
                                uint8_t* out, cudaStream_t stream) {
  t_err.clear();
  if (n < 0 || !valid_dtype(x_dtype) || !valid_blocksize(blocksize) ||
      (code_entries != 16 && code_entries != 256))
    return BQ_ERR_INVALID_ARG;
  if (n == 0) return BQ_OK;
  if (n > (int64_t{1} << 50)) return BQ_ERR_INVALID_ARG;
  const int eb = elem_bytes(x_dtype);
  if (!x || !code || !absmax || !out || !aligned(x, eb) || !aligned(absmax, 4) || !aligned(code, 4))
    return BQ_ERR_INVALID_ARG;

  int dev;
  DevInfo info;
  bq_status s = current_device(&dev, &info);
  if (s != BQ_OK) return s;

  bq::QParams p;
  p.x = x;
  p.n = n;
  p.code = code;
  p.absmax = absmax;
  p.out = out;
  p.bs = blocksize;
  p.nb = (n + blocksize - 1) / blocksize;
  p.full_tiles = 0;

  CUtensorMap map;
  std::memset(&map, 0, sizeof(map));
  const int64_t rows = n * eb / bq::kTileRows;             // whole 128-byte rows
  const int64_t tiles = rows / bq::kTileRows;              // whole 16 KiB tiles
  if (tiles > 0 && aligned(x, 16) && aligned(out, 16) && rows < (int64_t{1} << 31)) {
    PFN_cuTensorMapEncodeTiled_v12000 enc = encode_tiled();
    if (enc) {
      cuuint64_t dims[2] = {static_cast<cuuint64_t>(bq::kTileRows), static_cast<cuuint64_t>(rows)};
      cuuint64_t strides[1] = {static_cast<cuuint64_t>(bq::kTileRows)};
      cuuint32_t box[2] = {128, static_cast<cuuint32_t>(bq::kTileRows)};
      cuuint32_t estr[2] = {1, 1};
      CUresult r = enc(&map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(x), dims, strides,
                       box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                       CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
      if (r == CUDA_SUCCESS) p.full_tiles = tiles;
    }
  }

  switch (x_dtype) {
    case BQ_F32: return dispatch_quantize<bq::kF32>(p, code_entries, map, dev, info.sms, stream);
    case BQ_F16: return dispatch_quantize<bq::kF16>(p, code_entries, map, dev, info.sms, stream);
    default: return dispatch_quantize<bq::kBF16>(p, code_entries, map, dev, info.sms, stream);
  }
}

bq_status bq_dequantize_blockwise(const uint8_t* q, const float* absmax, int64_t n,
                                  int32_t blocksize, const float* code, int32_t code_entries,
                                  void* y, bq_dtype y_dtype, cudaStream_t stream) {
  t_err.clear();
  if (n < 0 || !valid_dtype(y_dtype) || !valid_blocksize(blocksize) ||
      (code_entries != 16 && code_entries != 256))
    return BQ_ERR_INVALID_ARG;
  if (n == 0) return BQ_OK;
  if (n > (int64_t{1} << 50)) return BQ_ERR_INVALID_ARG;
  if (!q || !absmax || !code || !y || !aligned(absmax, 4) || !aligned(code, 4) ||
      !aligned(y, elem_bytes(y_dtype)))
    return BQ_ERR_INVALID_ARG;
  bq::DParams p{};
  p.q = q;
  p.absmax = absmax;
  p.code = code;
  p.y = y;
  return dequant_entry<false>(p, n, blocksize, code_entries, y_dtype, stream);
}

bq_status bq_quantize_blockwise_nested(const void* x, bq_dtype x_dtype, int64_t n,
                                       int32_t blocksize, const float* code,
                                       int32_t code_entries, const float* code2,
                                       int32_t code2_entries, int32_t blocksize2, float* absmax,
                                       uint8_t* out, float* absmax2, uint8_t* qabsmax,
                                       cudaStream_t stream) {
  t_err.clear();
  if (n < 0 || !valid_dtype(x_dtype) || !valid_blocksize(blocksize) ||
      !valid_blocksize(blocksize2) || (code_entries != 16 && code_entries != 256) ||
      code2_entries != 256)
    return BQ_ERR_INVALID_ARG;
  if (n == 0) return BQ_OK;
  if (!code2 || !absmax2 || !qabsmax || !aligned(code2, 4) || !aligned(absmax2, 4))
    return BQ_ERR_INVALID_ARG;
  // the elements, then their fp32 statistics as a second blockwise input
  bq_status s = bq_quantize_blockwise(x, x_dtype, n, blocksize, code, code_entries, absmax, out,
                                      stream);
  if (s != BQ_OK) return s;
  const int64_t nb = (n + blocksize - 1) / blocksize;
  return bq_quantize_blockwise(absmax, BQ_F32, nb, blocksize2, code2, code2_entries, absmax2,
                               qabsmax, stream);
}

bq_status bq_quantize_blockwise_nested_noalloc(const void* x, bq_dtype x_dtype, int64_t n,
                                               int32_t blocksize, const float* code,
                                               int32_t code_entries, const float* code2,
                                               int32_t code2_entries, int32_t blocksize2,
                                               uint8_t* out, float* absmax2, uint8_t* qabsmax,
                                               cudaStream_t stream) {
  t_err.clear();
  if (n < 0 || !valid_dtype(x_dtype) || !valid_blocksize(blocksize) ||
      !valid_blocksize(blocksize2) || (code_entries != 16 && code_entries != 256) ||
      code2_entries != 256)
    return BQ_ERR_INVALID_ARG;
  if (n == 0) return BQ_OK;
  const int64_t nb = (n + blocksize - 1) / blocksize;
  if (nb > BQ_NOALLOC_MAX_BLOCKS) {
    t_err = "n / blocksize exceeds BQ_NOALLOC_MAX_BLOCKS (2^20 blocks): use "
            "bq_quantize_blockwise_nested with a caller-allocated absmax buffer";
    return BQ_ERR_INVALID_ARG;
  }
  int dev;
  DevInfo info;
  bq_status s = current_device(&dev, &info);
  if (s != BQ_OK) return s;
  float* stats = nullptr;
  s = noalloc_stats(dev, &stats);
  if (s != BQ_OK) return s;
  return bq_quantize_blockwise_nested(x, x_dtype, n, blocksize, code, code_entries, code2,
                                      code2_entries, blocksize2, stats, out, absmax2, qabsmax,
                                      stream);
}

bq_status bq_dequantize_blockwise_nested(const uint8_t* q, const uint8_t* qabsmax,
                                         const float* absmax2, int64_t n, int32_t blocksize,
                                         const float* code, int32_t code_entries,
                                         const float* code2, int32_t code2_entries,
                                         int32_t blocksize2, void* y, bq_dtype y_dtype,
                                         cudaStream_t stream) {
  t_err.clear();
  if (n < 0 || !valid_dtype(y_dtype) || !valid_blocksize(blocksize) ||
      !valid_blocksize(blocksize2) || (code_entries != 16 && code_entries != 256) ||
      code2_entries != 256)
    return BQ_ERR_INVALID_ARG;
  if (n == 0) return BQ_OK;
  if (n > (int64_t{1} << 50)) return BQ_ERR_INVALID_ARG;
  if (!q || !qabsmax || !absmax2 || !code || !code2 || !y || !aligned(absmax2, 4) ||
      !aligned(code, 4) || !aligned(code2, 4) || !aligned(y, elem_bytes(y_dtype)))
    return BQ_ERR_INVALID_ARG;
  bq::DParams p{};
  p.q = q;
  p.code = code;
  p.y = y;
  p.qa = qabsmax;
  p.absmax2 = absmax2;
  p.code2 = code2;
  p.bs2_log2 = log2i(blocksize2);
  return dequant_entry<true>(p, n, blocksize, code_entries, y_dtype, stream);
}

bq_status bq_quantize_blockwise_host(const void* x_host, bq_dtype x_dtype, int64_t n,
                                     int32_t blocksize, const float* code, int32_t code_entries,
                                     const float* code2, int32_t code2_entries,
                                     int32_t blocksize2, float* absmax, uint8_t* out,
                                     float* absmax2, uint8_t* qabsmax, void* staging,
                                     int64_t staging_bytes, int64_t chunk_elements,
                                     cudaStream_t stream0, cudaStream_t stream1) {
  t_err.clear();
  const bool nested = code2 != nullptr;
  if (n < 0 || !valid_dtype(x_dtype) || !valid_blocksize(blocksize) ||
      (code_entries != 16 && code_entries != 256))
    return BQ_ERR_INVALID_ARG;
  if (nested && (!valid_blocksize(blocksize2) || code2_entries != 256 || !absmax2 || !qabsmax))
    return BQ_ERR_INVALID_ARG;
  // chunks are whole blocks (whole second-level blocks with compressed
  // statistics), so every chunk's outputs start where the whole call's would
  const int64_t unit = nested ? int64_t{blocksize} * blocksize2 : blocksize;
  if (chunk_elements <= 0 || chunk_elements % unit != 0 || chunk_elements > (int64_t{1} << 40))
    return BQ_ERR_INVALID_ARG;
  if (n == 0) return BQ_OK;
  const int eb = elem_bytes(x_dtype);
  const int64_t chunks = (n + chunk_elements - 1) / chunk_elements;
  const int64_t chunk_bytes = chunk_elements * eb;
  const int64_t need = chunks > 1 ? 2 * chunk_bytes : n * eb;
  if (!x_host || !aligned(x_host, eb) || !staging || !aligned(staging, 16) ||
      staging_bytes < need || !absmax || !out)
    return BQ_ERR_INVALID_ARG;

  cudaEvent_t joined = nullptr;
  const bool two = chunks > 1 && stream1 != stream0;
  if (two) {
    cudaError_t e = cudaEventCreateWithFlags(&joined, cudaEventDisableTiming);
    if (e != cudaSuccess) return cuda_fail(e, "pipeline event");
    // stream1's chunks start only after the work already queued on stream0
    // (which may still use the outputs or the staging buffer)
    e = cudaEventRecord(joined, stream0);
    if (e == cudaSuccess) e = cudaStreamWaitEvent(stream1, joined, 0);
    if (e != cudaSuccess) {
      cudaEventDestroy(joined);
      return cuda_fail(e, "pipeline entry ordering");
    }
  }
  bq_status st = BQ_OK;
  for (int64_t i = 0; i < chunks && st == BQ_OK; ++i) {
    // chunk i goes to staging half i % 2 on stream i % 2: the copy of one
    // chunk overlaps the quantization of the other, and a half is refilled
    // only after the quantization that read it (same stream)
    const int64_t off = i * chunk_elements;
    const int64_t len = n - off < chunk_elements ? n - off : chunk_elements;
    cudaStream_t s = (i & 1) ? stream1 : stream0;
    void* dst = static_cast<uint8_t*>(staging) + (i & 1) * chunk_bytes;
    cudaError_t e = cudaMemcpyAsync(dst, static_cast<const uint8_t*>(x_host) + off * eb,
                                    static_cast<size_t>(len * eb), cudaMemcpyHostToDevice, s);
    if (e != cudaSuccess) {
      st = cuda_fail(e, "pipeline host-to-device copy");
      break;
    }
    const int64_t b0 = off / blocksize;
    uint8_t* o = out + (code_entries == 16 ? off / 2 : off);
    st = nested ? bq_quantize_blockwise_nested(dst, x_dtype, len, blocksize, code, code_entries,
                                               code2, code2_entries, blocksize2, absmax + b0, o,
                                               absmax2 + b0 / blocksize2, qabsmax + b0, s)
                : bq_quantize_blockwise(dst, x_dtype, len, blocksize, code, code_entries,
                                        absmax + b0, o, s);
  }
  if (two) {
    // stream0 continues only after stream1's chunks (the event is re-recorded:
    // cudaStreamWaitEvent above captured its first recording already)
    cudaError_t e = cudaEventRecord(joined, stream1);
    if (e == cudaSuccess) e = cudaStreamWaitEvent(stream0, joined, 0);
    if (e != cudaSuccess && st == BQ_OK) st = cuda_fail(e, "pipeline join");
    cudaEventDestroy(joined);  // released once the recorded work completes
  }
  return st;
}

bq_status bq_dequant_q8_0(const void* blocks, int64_t n_blocks, void* y, bq_dtype y_dtype,
                          cudaStream_t stream) {
  return gguf_entry<bq::kQ8_0>(blocks, n_blocks, y, y_dtype, stream);
}

bq_status bq_dequant_q4_0(const void* blocks, int64_t n_blocks, void* y, bq_dtype y_dtype,
                          cudaStream_t stream) {
  return gguf_entry<bq::kQ4_0>(blocks, n_blocks, y, y_dtype, stream);
}

bq_status bq_dequant_q4_1(const void* blocks, int64_t n_blocks, void* y, bq_dtype y_dtype,
                          cudaStream_t stream) {
  return gguf_entry<bq::kQ4_1>(blocks, n_blocks, y, y_dtype, stream);
}

bq_status bq_dequant_q5_0(const void* blocks, int64_t n_blocks, void* y, bq_dtype y_dtype,
                          cudaStream_t stream) {
  return gguf_entry<bq::kQ5_0>(blocks, n_blocks, y, y_dtype, stream);
}

bq_status bq_dequant_q5_1(const void* blocks, int64_t n_blocks, void* y, bq_dtype y_dtype,
                          cudaStream_t stream) {
  return gguf_entry<bq::kQ5_1>(blocks, n_blocks, y, y_dtype, stream);
}

bq_status bq_dequant_q4_k(const void* blocks, int64_t n_blocks, void* y, bq_dtype y_dtype,
                          cudaStream_t stream) {
  return gguf_entry<bq::kQ4_K>(blocks, n_blocks, y, y_dtype, stream);
}

bq_status bq_dequant_q6_k(const void* blocks, int64_t n_blocks, void* y, bq_dtype y_dtype,
                          cudaStream_t stream) {
  return gguf_entry<bq::kQ6_K>(blocks, n_blocks, y, y_dtype, stream);
}

bq_status bq_dequant_q2_k(const void* blocks, int64_t n_blocks, void* y, bq_dtype y_dtype,
                          cudaStream_t stream) {
  return gguf_entry<bq::kQ2_K>(blocks, n_blocks, y, y_dtype, stream);
}

bq_status bq_dequant_q3_k(const void* blocks, int64_t n_blocks, void* y, bq_dtype y_dtype,
                          cudaStream_t stream) {
  return gguf_entry<bq::kQ3_K>(blocks, n_blocks, y, y_dtype, stream);
}

bq_status bq_dequant_q5_k(const void* blocks, int64_t n_blocks, void* y, bq_dtype y_dtype,
                          cudaStream_t stream) {
  return gguf_entry<bq::kQ5_K>(blocks, n_blocks, y, y_dtype, stream);
}

bq_status bq_dequant_bf16(const void* x, int64_t n, void* y, bq_dtype y_dtype,
                          cudaStream_t stream) {
  t_err.clear();
  if (n < 0 || !valid_dtype(y_dtype)) return BQ_ERR_INVALID_ARG;
  if (n == 0) return BQ_OK;
  if (n > (int64_t{1} << 56)) return BQ_ERR_INVALID_ARG;
  if (!x || !y || !aligned(x, 2) || !aligned(y, elem_bytes(y_dtype))) return BQ_ERR_INVALID_ARG;
  int dev;
  DevInfo info;
  bq_status s = current_device(&dev, &info);
  if (s != BQ_OK) return s;
  bq::BParams p;
  p.x = static_cast<const uint16_t*>(x);
  p.y = y;
  p.n = n;
  p.ngroups = aligned(x, 16) && aligned(y, 16) ? n / 8 : 0;
  switch (y_dtype) {
    case BQ_F32: return launch_bf16<bq::kF32>(p, dev, info.sms, stream);
    case BQ_F16: return launch_bf16<bq::kF16>(p, dev, info.sms, stream);
    default: return launch_bf16<bq::kBF16>(p, dev, info.sms, stream);
  }
}

bq_status bq_quantize_q8_0(const void* x, bq_dtype x_dtype, int64_t n, void* blocks,
                           cudaStream_t stream) {
  return gguf_encode_entry<bq::kQ8_0>(x, x_dtype, n, blocks, stream);
}

bq_status bq_quantize_q4_0(const void* x, bq_dtype x_dtype, int64_t n, void* blocks,
                           cudaStream_t stream) {
  return gguf_encode_entry<bq::kQ4_0>(x, x_dtype, n, blocks, stream);
}

const char* bq_status_string(bq_status s) {
  switch (s) {
    case BQ_OK: return "ok";
    case BQ_ERR_INVALID_ARG: return "invalid argument";
    case BQ_ERR_UNSUPPORTED: return "unsupported";
    case BQ_ERR_CUDA: return "CUDA error";
    default: return "unknown status";
  }
}

const char* bq_last_cuda_error(void) { return t_err.c_str(); }

bq_status bq_device_fault(uint32_t* fault, int32_t reset) {
  t_err.clear();
  if (!fault) return BQ_ERR_INVALID_ARG;
  uint32_t v = 0;
  cudaError_t e = cudaMemcpyFromSymbol(&v, bq::g_fault, sizeof(v));
  if (e != cudaSuccess) return cuda_fail(e, "reading the fault word");
  *fault = v;
  if (reset) {
    const uint32_t zero = 0;
    e = cudaMemcpyToSymbol(bq::g_fault, &zero, sizeof(zero));
    if (e != cudaSuccess) return cuda_fail(e, "clearing the fault word");
  }
  return BQ_OK;
}

int32_t bq_abi_version(void) { return BQ_ABI_VERSION; }

#ifdef BQ_TEST_HOOKS
// Test builds only (not declared in bq.h, not in libbq.so): choose the tile
// whose copy the pipelined kernels' producers skip (-1: none).
__attribute__((visibility("default"))) bq_status bq_test_skip_tile(int64_t tile) {
  const cudaError_t e = cudaMemcpyToSymbol(bq::g_test_skip_tile, &tile, sizeof(tile));
  return e == cudaSuccess ? BQ_OK : cuda_fail(e, "setting the test hook");
}
#endif

}  // extern "C"
