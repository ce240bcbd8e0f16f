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
// host-side stand-in, so the device address is looked up with cudaGetSymbolAddress, once per device,
// with that device current, on the first call made on that device.
#include <mutex>

#include "common.cuh"

namespace pisa {
namespace {

constexpr size_t kNoAllocScratchBytes = size_t(16) << 20;   // 16 MiB
constexpr int kMaxDevices = 64;

__device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

std::mutex g_mu;
void* g_scratch_addr[kMaxDevices] = {};

// Device address of g_noalloc_scratch on the current device (looked up once per device).
cudaError_t scratch_address(void** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lock(g_mu);
  if (!g_scratch_addr[dev]) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
    if (e != cudaSuccess) return e;
    g_scratch_addr[dev] = p;
  }
  *out = g_scratch_addr[dev];
  return cudaSuccess;
}

}  // namespace
}  // namespace pisa

extern "C" pisa_status pisa_precompute_noalloc(const pisa_shape* shape, const void* q, const void* k, const void* v,
                                               const pisa_stats* stats, pisa_stream_t stream) {
  const size_t need = pisa_workspace_bytes(shape);
  if (need == 0) {
    // same validation as pisa_precompute, which reports the precise status
    return pisa_precompute(shape, q, k, v, stats, nullptr, 0, stream);
  }
  if (need > pisa::kNoAllocScratchBytes) return PISA_ERR_UNSUPPORTED;
  void* ws = nullptr;
  if (pisa::scratch_address(&ws) != cudaSuccess) return PISA_ERR_CUDA;
  cudaStream_t cs = reinterpret_cast<cudaStream_t>(stream);
  // the device status word at the start of the scratch must be zero when the kernels start
  if (cudaMemsetAsync(ws, 0, pisa::kStatusBytes, cs) != cudaSuccess) return PISA_ERR_CUDA;
  return pisa_precompute(shape, q, k, v, stats, ws, need, stream);
}
