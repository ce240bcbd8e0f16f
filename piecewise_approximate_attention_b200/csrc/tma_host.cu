// Host-side helpers: TMA descriptor encoding (cuTensorMapEncodeTiled through the runtime's driver
// entry point, so the library needs no link-time dependency on libcuda), the kernels'
// dynamic-shared-memory attribute, set once per kernel and device, and the device's SM count.
#include <cudaTypedefs.h>

#include <atomic>
#include <map>
#include <mutex>
#include <utility>

#include "common.cuh"

namespace pisa {
namespace {

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q = cudaDriverEntryPointSymbolNotFound;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(ptr);
  });
  return fn;
}

std::mutex g_attr_mu;
// (kernel, CUDA context id) -> bytes already allowed; keyed by context so that a context created
// after cudaDeviceReset sets the attribute again
std::map<std::pair<const void*, unsigned long long>, size_t> g_attr_set;

}  // namespace

// Unique id of the calling thread's current CUDA context (0 if none is current or the driver
// cannot say).  Driver entry points through the runtime: no link-time dependency on libcuda.
unsigned long long current_context_id() {
  static PFN_cuCtxGetCurrent_v4000 get_cur = nullptr;
  static PFN_cuCtxGetId_v12000 get_id = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q = cudaDriverEntryPointSymbolNotFound;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      get_cur = reinterpret_cast<PFN_cuCtxGetCurrent_v4000>(p);
    p = nullptr;
    if (cudaGetDriverEntryPoint("cuCtxGetId", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      get_id = reinterpret_cast<PFN_cuCtxGetId_v12000>(p);
  });
  if (!get_cur || !get_id) return 0;
  CUcontext ctx = nullptr;
  unsigned long long id = 0;
  if (get_cur(&ctx) != CUDA_SUCCESS || !ctx || get_id(ctx, &id) != CUDA_SUCCESS) return 0;
  return id;
}

cudaError_t sm_count(int* n) {
  static std::atomic<int> cache[64];     // per device ordinal; 0 = not asked yet
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  const bool cached = dev >= 0 && dev < 64;
  if (cached && (*n = cache[dev].load(std::memory_order_relaxed)) > 0) return cudaSuccess;
  if ((e = cudaDeviceGetAttribute(n, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess) return e;
  if (cached) cache[dev].store(*n, std::memory_order_relaxed);
  return cudaSuccess;
}

cudaError_t set_max_dynamic_smem(const void* fn, size_t bytes) {
  const unsigned long long ctx = current_context_id();
  std::lock_guard<std::mutex> lock(g_attr_mu);
  if (ctx != 0) {
    auto it = g_attr_set.find({fn, ctx});
    if (it != g_attr_set.end() && it->second >= bytes) return cudaSuccess;
  }
  const cudaError_t e = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes);
  if (e != cudaSuccess) return e;
  if (ctx != 0) g_attr_set[{fn, ctx}] = bytes;
  return cudaSuccess;
}

bool encode_bf16_3d(CUtensorMap* map, const void* base, uint64_t inner, uint64_t rows, uint64_t batch,
                    uint32_t box_rows) {
  return encode_16bit_3d(map, base, inner, rows, batch, box_rows, false);
}

bool encode_16bit_3d(CUtensorMap* map, const void* base, uint64_t inner, uint64_t rows, uint64_t batch,
                     uint32_t box_rows, bool fp16) {
  auto fn = encode_fn();
  if (!fn || !base) return false;
  cuuint64_t dims[3] = {inner, rows, batch};
  cuuint64_t strides[2] = {inner * 2, rows * inner * 2};
  cuuint32_t box[3] = {64, box_rows, 1};
  cuuint32_t estride[3] = {1, 1, 1};
  const CUresult r = fn(map, fp16 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT16 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box, estride,
                        CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                        CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

bool encode_u8_3d(CUtensorMap* map, const void* base, uint64_t inner, uint64_t rows, uint64_t batch,
                  uint32_t box_rows) {
  auto fn = encode_fn();
  if (!fn || !base || inner != 128) return false;
  cuuint64_t dims[3] = {inner, rows, batch};
  cuuint64_t strides[2] = {inner, rows * inner};
  cuuint32_t box[3] = {128, box_rows, 1};
  cuuint32_t estride[3] = {1, 1, 1};
  const CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, const_cast<void*>(base), dims, strides, box, estride,
                        CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                        CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

}  // namespace pisa
