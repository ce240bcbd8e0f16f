// Shared device/host definitions of the PISA library (internal; not part of the C ABI).
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <stdint.h>

#include "pisa.h"

namespace pisa {

// Problem dimensions after validation.
struct Dims {
  int B, H, L, d, block, nb, dtype;
  float scale;
  int BH() const { return B * H; }
  int last_cnt() const { return L - (nb - 1) * block; }
};

// Workspace layout: [0, 256) device status word(s); [256, ...) precompute partial sums of H_j.
constexpr size_t kStatusBytes = 256;
constexpr int kBlocksPerPart = 16;   // key blocks whose H_j one precompute CTA sums

inline int num_parts(const Dims& g) { return (g.nb + kBlocksPerPart - 1) / kBlocksPerPart; }
inline size_t partials_bytes(const Dims& g) {
  return (size_t)g.BH() * num_parts(g) * g.d * g.d * sizeof(float);
}
// after the partials: per (head, group of blocks) max |v|, which sets the head's value scale
inline size_t vmax_bytes(const Dims& g) { return (size_t)g.BH() * num_parts(g) * sizeof(float); }
inline size_t vmax_offset(const Dims& g) { return kStatusBytes + ((partials_bytes(g) + 255) / 256) * 256; }
// per-block first-order mode: per query row (softmax offset in log2 units, 1 / D_t) at kStatusBytes,
// then the attention output in fp32 (rounded to bf16 once, after the per-block term is added)
inline size_t rowstats_bytes(const Dims& g) { return (size_t)g.BH() * g.L * 2 * sizeof(float); }
inline size_t o32_offset(const Dims& g) { return kStatusBytes + (rowstats_bytes(g) + 255) / 256 * 256; }
inline size_t perblock_ws_bytes(const Dims& g) { return o32_offset(g) + (size_t)g.BH() * g.L * g.d * sizeof(float); }

__device__ __forceinline__ float to_f32(float x) { return x; }
__device__ __forceinline__ float to_f32(__nv_bfloat16 x) { return __bfloat162float(x); }
template <typename T> __device__ __forceinline__ T from_f32(float x);
template <> __device__ __forceinline__ float from_f32<float>(float x) { return x; }
template <> __device__ __forceinline__ __nv_bfloat16 from_f32<__nv_bfloat16>(float x) {
  return __float2bfloat16_rn(x);
}

// Records the first device-side error code; later codes do not overwrite it.
__device__ __forceinline__ void set_status(int* status, int code) {
  if (status) atomicCAS(status, 0, code);
}

__device__ __forceinline__ int block_count(int j, int L, int block) {
  int s = j * block;
  int e = s + block < L ? s + block : L;
  return e - s;
}

// Inputs stored as bf16 (PISA_BF16, and PISA_BF16_FP8QK whose logits use e4m3 copies).
inline bool bf16_inputs(int dtype) { return dtype == PISA_BF16 || dtype == PISA_BF16_FP8QK; }

// TMA descriptors of one pisa_attention call (bf16 inputs); q8, k8, kbar8 only for e4m3 logits.
struct AttnMaps {
  CUtensorMap q, k, v, kbar, vsum, hbar;
  CUtensorMap q8, k8, kbar8;
};

// Scales of the e4m3 operand copies (all null on the bf16 path): per query row [B*H][L], per key
// block [B*H][nb], per tile of 128 centroids [B*H][ceil(nb/128)].
struct F8Scales {
  const float* q = nullptr;
  const float* k = nullptr;
  const float* kb = nullptr;
};

// Encodes a 3-D bf16 tensor [batch][rows][inner] (row-major) with a {64, box_rows, 1} box and
// 128-byte swizzling; false if the driver entry point is unavailable or rejects the arguments.
bool encode_bf16_3d(CUtensorMap* map, const void* base, uint64_t inner, uint64_t rows, uint64_t batch,
                    uint32_t box_rows);
// Same for a bf16 (fp16 == false) or fp16 (fp16 == true) tensor.
bool encode_16bit_3d(CUtensorMap* map, const void* base, uint64_t inner, uint64_t rows, uint64_t batch,
                     uint32_t box_rows, bool fp16);
// A 3-D byte tensor [batch][rows][128] with a {128, box_rows, 1} box and 128-byte swizzling (e4m3).
bool encode_u8_3d(CUtensorMap* map, const void* base, uint64_t inner, uint64_t rows, uint64_t batch,
                  uint32_t box_rows);

constexpr unsigned long long kWaitLimitNs = 2000000000ull;   // bounded mbarrier waits: 2 s

// cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes) on the current
// device, made only when this kernel has not yet been given at least `bytes` there: the driver
// call would otherwise be repeated, on the host, before every launch.
cudaError_t set_max_dynamic_smem(const void* fn, size_t bytes);

// Unique id of the calling thread's current CUDA context, 0 if none is current (or the driver
// cannot say).  Host caches of per-context state key on it.
unsigned long long current_context_id();
// Number of SMs of the current device (cached per device ordinal).
cudaError_t sm_count(int* n);

// Argument checks of pisa_precompute other than its workspace (shape, q, k, v, stats); fills *g.
// Enqueues nothing.  Shared by the entry points that run the pre-computation.
pisa_status validate_precompute(const pisa_shape* shape, const void* q, const void* k, const void* v,
                                const pisa_stats* stats, Dims* g);

// ---- launchers (defined in the kernel translation units) ----
// first_order = false: the zeroth-order statistics only (pisa_precompute_zeroth_order).
cudaError_t launch_precompute_simt(const Dims& g, const void* q, const void* k, const void* v,
                                   const pisa_stats& st, void* ws, bool first_order, cudaStream_t stream);
// wait_ns: the kernels' bounded-wait limit; fault: test-only fault injection (pisa_testing.h), 0
// in normal calls.
cudaError_t launch_precompute_sm100(const Dims& g, const void* q, const void* k, const void* v,
                                    const pisa_stats& st, void* ws, bool first_order,
                                    unsigned long long wait_ns, int fault, cudaStream_t stream);
// pdl: launch with programmatic stream serialization (the kernel waits for the previous kernel of
// the stream before it reads anything, and lets the next one start at once).
cudaError_t launch_hbar_reduce(const Dims& g, const float* partials, int nparts, const float* vmax,
                               const pisa_stats& st, cudaStream_t stream, bool pdl = false);
cudaError_t launch_route(const Dims& g, const pisa_stats& st, int keep_k, float lam, int32_t* sel,
                         int32_t* order, float* scores, cudaStream_t stream);
// Pre-computation + routing in one cluster launch (bf16 inputs, d = 128, nb <= 128).  *launched is
// false (and nothing is enqueued) when the shape is not eligible or the device cannot schedule the
// cluster; the caller then runs the separate kernels.
bool short_step_eligible(const Dims& g);
cudaError_t launch_short_step_sm100(const Dims& g, const void* q, const void* k, const void* v, const pisa_stats& st,
                                    void* ws, int keep_k, float lam, int32_t* sel, int32_t* order, float* scores,
                                    cudaStream_t stream, bool* launched);
cudaError_t launch_attention_sm100(const Dims& g, const AttnMaps& maps, const int32_t* sel, const int32_t* order,
                                   int keep_k, int mode, const float* vscale, const F8Scales& f8, void* o,
                                   float2* rowstats, float* o32, int* status, unsigned long long wait_ns, int fault,
                                   cudaStream_t stream);
cudaError_t launch_quantize_fp8(const Dims& g, const void* q, const void* k, const pisa_stats& st, cudaStream_t stream);
cudaError_t launch_permute_rows(const void* src, void* dst, const int32_t* perm, int batch_heads, int L,
                                int row_bytes, int perm_per_head, int inverse, cudaStream_t stream);
cudaError_t launch_perblock_sm100(const Dims& g, const AttnMaps& maps, const CUtensorMap& hdiff,
                                  const int32_t* sel, const int32_t* order, int keep_k, const float2* rowstats,
                                  const float* o32, void* o, int* status, unsigned long long wait_ns,
                                  cudaStream_t stream);
cudaError_t launch_attention_simt(const Dims& g, const void* q, const void* k, const void* v,
                                  const pisa_stats& st, const int32_t* sel, int keep_k, int mode,
                                  void* o, int* status, cudaStream_t stream);

}  // namespace pisa
