// e4m3 operand copies for logits on the tensor core in PISA_BF16_FP8QK mode: q with one scale per
// row, k with one scale per key block, kbar with one scale per tile of 128 centroids.  A group's
// scale is max|x| / 448 (1 for an all-zero group) and the code of x is e4m3(x / scale), rounded to
// nearest even and saturated, both computed in float32 (IEEE division).
//
// HBM-bound: q and k are read once more (bf16) and written as one byte per element.  One warp per
// row, four elements per lane (a 128-element row is 256 bytes of bf16 in, 128 bytes of codes out);
// a warp issues the loads of several rows before it reduces any of them, so that enough bytes are
// in flight to cover the memory latency.
#include "common.cuh"

namespace pisa {
namespace {

constexpr int kThreads = 256;
constexpr int kWarps = kThreads / 32;
constexpr int kRowsPerWarp = 4;
constexpr float kE4m3Max = 448.f;

__device__ __forceinline__ uint16_t pack_e4m3x2(float lo, float hi) {
  uint16_t r;
  asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(hi), "f"(lo));
  return r;
}

// Four consecutive elements of a row as float32, from bf16 or float32 storage.
__device__ __forceinline__ void load4(const __nv_bfloat16* row, int lane, float* x) {
  const uint2 u = *reinterpret_cast<const uint2*>(row + 4 * lane);
  x[0] = __uint_as_float(u.x << 16);
  x[1] = __uint_as_float(u.x & 0xffff0000u);
  x[2] = __uint_as_float(u.y << 16);
  x[3] = __uint_as_float(u.y & 0xffff0000u);
}
__device__ __forceinline__ void load4(const float* row, int lane, float* x) {
  const float4 u = *reinterpret_cast<const float4*>(row + 4 * lane);
  x[0] = u.x;
  x[1] = u.y;
  x[2] = u.z;
  x[3] = u.w;
}

__device__ __forceinline__ float warp_absmax(const float* x) {
  const float m = fmaxf(fmaxf(fabsf(x[0]), fabsf(x[1])), fmaxf(fabsf(x[2]), fabsf(x[3])));
  // non-negative floats order like their bit patterns
  return __uint_as_float(__reduce_max_sync(0xffffffffu, __float_as_uint(m)));
}

__device__ __forceinline__ void store_codes(uint8_t* row, int lane, const float* x, float s) {
  const uint32_t c = (uint32_t)pack_e4m3x2(x[0] / s, x[1] / s) | ((uint32_t)pack_e4m3x2(x[2] / s, x[3] / s) << 16);
  *reinterpret_cast<uint32_t*>(row + 4 * lane) = c;
}

// One scale per row: rows of [B*H][L][128] bf16.
__global__ void __launch_bounds__(kThreads) quant_rows(const __nv_bfloat16* __restrict__ src, uint8_t* __restrict__ dst,
                                                      float* __restrict__ scale, int L) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, bh = blockIdx.y;
  const int r0 = (blockIdx.x * kWarps + warp) * kRowsPerWarp;
  float x[kRowsPerWarp][4];
#pragma unroll
  for (int e = 0; e < kRowsPerWarp; ++e)
    if (r0 + e < L) load4(src + ((size_t)bh * L + r0 + e) * 128, lane, x[e]);
#pragma unroll
  for (int e = 0; e < kRowsPerWarp; ++e) {
    if (r0 + e >= L) break;
    const size_t row = (size_t)bh * L + r0 + e;
    const float amax = warp_absmax(x[e]);
    const float s = amax > 0.f ? amax / kE4m3Max : 1.f;
    store_codes(dst + row * 128, lane, x[e], s);
    if (lane == 0) scale[row] = s;
  }
}

// One scale per group of `group` consecutive rows (key blocks, or tiles of 128 centroids).
template <typename T>
__global__ void __launch_bounds__(kThreads) quant_groups(const T* __restrict__ src, uint8_t* __restrict__ dst,
                                                        float* __restrict__ scale, int rows, int group) {
  __shared__ float red[kWarps];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, bh = blockIdx.y;
  const int r0 = blockIdx.x * group, r1 = min(rows, r0 + group);
  const size_t base = (size_t)bh * rows;
  float m = 0.f;
  // the maximum over the group's rows, four rows of a warp in flight at once
  for (int r = r0 + warp; r < r1; r += 4 * kWarps) {
    float x[4][4];
#pragma unroll
    for (int e = 0; e < 4; ++e)
      if (r + e * kWarps < r1) load4(src + (base + r + e * kWarps) * 128, lane, x[e]);
#pragma unroll
    for (int e = 0; e < 4; ++e)
      if (r + e * kWarps < r1) m = fmaxf(m, warp_absmax(x[e]));
  }
  if (lane == 0) red[warp] = m;
  __syncthreads();
  float amax = 0.f;
  for (int w = 0; w < kWarps; ++w) amax = fmaxf(amax, red[w]);
  const float s = amax > 0.f ? amax / kE4m3Max : 1.f;
  for (int r = r0 + warp; r < r1; r += 4 * kWarps) {
    float x[4][4];
#pragma unroll
    for (int e = 0; e < 4; ++e)
      if (r + e * kWarps < r1) load4(src + (base + r + e * kWarps) * 128, lane, x[e]);
#pragma unroll
    for (int e = 0; e < 4; ++e)
      if (r + e * kWarps < r1) store_codes(dst + (base + r + e * kWarps) * 128, lane, x[e], s);
  }
  if (threadIdx.x == 0) scale[(size_t)bh * gridDim.x + blockIdx.x] = s;
}

}  // namespace

cudaError_t launch_quantize_fp8(const Dims& g, const void* q, const void* k, const pisa_stats& st, cudaStream_t stream) {
  const int rows_per_cta = kWarps * kRowsPerWarp;
  quant_rows<<<dim3((g.L + rows_per_cta - 1) / rows_per_cta, g.BH()), kThreads, 0, stream>>>(
      static_cast<const __nv_bfloat16*>(q), static_cast<uint8_t*>(st.q8), st.qscale, g.L);
  quant_groups<__nv_bfloat16><<<dim3(g.nb, g.BH()), kThreads, 0, stream>>>(
      static_cast<const __nv_bfloat16*>(k), static_cast<uint8_t*>(st.k8), st.kscale, g.L, g.block);
  quant_groups<float><<<dim3((g.nb + 127) / 128, g.BH()), kThreads, 0, stream>>>(
      st.kbar, static_cast<uint8_t*>(st.kbar8), st.kbscale, g.nb, 128);
  return cudaGetLastError();
}

}  // namespace pisa
