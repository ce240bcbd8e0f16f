// pisa_precompute_noalloc: the pre-computation for callers that cannot allocate device memory.
//
// Some callers have no way to obtain scratch memory: a plugin running inside a host framework that
// owns every device allocation and hands the plugin only its inputs and outputs, or a latency-critical
// path that must not call cudaMalloc (which can synchronise the whole device).  For them this entry
// point runs the same pre-computation kernels as pisa_precompute, with the workspace taken from a
// fixed array in the library's own device memory instead of a caller buffer.
//
// The array is a file-scope __device__ variable of kNoAllocScratchBytes.  Every device on which the
// library's module is loaded holds it until the process exits.  In host code its name is only a
// host-side stand-in, so its device address is looked up with cudaGetSymbolAddress, with the device
// current, the first time a call runs in a device's CUDA context (and again if that context has been
// replaced, e.g. after cudaDeviceReset, since the module is then loaded afresh).
#include <mutex>

#include "common.cuh"

namespace pisa {
namespace {

constexpr size_t kNoAllocScratchBytes = size_t(16) << 20;   // 16 MiB
constexpr int kMaxDevices = 64;

__device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

std::mutex g_mu;
struct ScratchEntry {
  unsigned long long ctx_id = 0;   // CUDA context the address belongs to (0 = not looked up yet)
  void* addr = nullptr;
};
ScratchEntry g_scratch[kMaxDevices];

// Device address of g_noalloc_scratch in the current device's context.  Looked up once per
// context; a host-side query that allocates nothing.
cudaError_t scratch_address(void** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lock(g_mu);
  ScratchEntry& ent = g_scratch[dev];
  const unsigned long long id = current_context_id();
  if (!ent.addr || id == 0 || id != ent.ctx_id) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
    if (e != cudaSuccess) return e;
    ent.addr = p;
    // the lookup makes the device's context current if it was not: ask again for its id
    ent.ctx_id = id ? id : current_context_id();
  }
  *out = ent.addr;
  return cudaSuccess;
}

}  // namespace
}  // namespace pisa

extern "C" pisa_status pisa_precompute_noalloc(const pisa_shape* shape, const void* q, const void* k, const void* v,
                                               const pisa_stats* stats, pisa_stream_t stream) {
  // every check pisa_precompute makes (apart from its workspace) comes first: a rejected call
  // enqueues nothing and leaves the shared scratch alone
  pisa::Dims g;
  const pisa_status s = pisa::validate_precompute(shape, q, k, v, stats, &g);
  if (s != PISA_OK) return s;
  const size_t need = pisa_workspace_bytes(shape);
  if (need == 0) return PISA_ERR_INVALID_ARG;
  if (need > pisa::kNoAllocScratchBytes) return PISA_ERR_UNSUPPORTED;
  void* ws = nullptr;
  if (pisa::scratch_address(&ws) != cudaSuccess) return PISA_ERR_CUDA;
  cudaStream_t cs = reinterpret_cast<cudaStream_t>(stream);
  // the device status word at the start of the scratch must be zero when the kernels start
  if (cudaMemsetAsync(ws, 0, pisa::kStatusBytes, cs) != cudaSuccess) return PISA_ERR_CUDA;
  return pisa_precompute(shape, q, k, v, stats, ws, need, stream);
}
