// Token reordering before blocking (PAROAttention, "Pattern-Aware ReOrdering", abstract): rows of
// a [B*H][L][row_bytes] tensor are gathered through a permutation (dst[i] = src[perm[i]]) or
// scattered back with its inverse (dst[perm[i]] = src[i]), so that the blocks PISA forms over the
// reordered sequence follow another axis order of the video's (frames, height, width) grid.
//
// HBM-bound copy: every row is read once and written once as 16-byte vectors; consecutive threads
// take consecutive 16-byte chunks of a row, so each warp moves whole rows with full sectors.
// The grid is sized to a few CTAs per SM and strides over the rows.
#include "common.cuh"

namespace pisa {
namespace {

constexpr int kThreads = 256;
constexpr int kUnroll = 4;

__global__ void __launch_bounds__(kThreads) permute_rows_kernel(const uint4* __restrict__ src, uint4* __restrict__ dst,
                                                                const int32_t* __restrict__ perm, int L,
                                                                int chunks, int perm_per_head, int inverse,
                                                                long long total) {
  const int bh = blockIdx.y;
  const int32_t* pr = perm + (perm_per_head ? (size_t)bh * L : 0);
  const size_t base = (size_t)bh * L * chunks;
  const long long stride = (long long)gridDim.x * kThreads;
  // kUnroll chunks per thread per round: all loads are issued before the stores
  for (long long e0 = (long long)blockIdx.x * kThreads + threadIdx.x; e0 < total; e0 += kUnroll * stride) {
    uint4 val[kUnroll];
    size_t to[kUnroll];
    bool ok[kUnroll];
#pragma unroll
    for (int u = 0; u < kUnroll; ++u) {
      const long long e = e0 + u * stride;
      ok[u] = false;
      if (e < total) {
        const int i = (int)(e / chunks), c = (int)(e % chunks);
        const int j = pr[i];
        if (j >= 0 && j < L) {   // out-of-range entries are skipped (documented in pisa.h)
          const size_t from = inverse ? (size_t)i : (size_t)j;
          to[u] = base + (inverse ? (size_t)j : (size_t)i) * chunks + c;
          val[u] = src[base + from * chunks + c];
          ok[u] = true;
        }
      }
    }
#pragma unroll
    for (int u = 0; u < kUnroll; ++u)
      if (ok[u]) dst[to[u]] = val[u];
  }
}

}  // namespace

cudaError_t launch_permute_rows(const void* src, void* dst, const int32_t* perm, int batch_heads, int L,
                                int row_bytes, int perm_per_head, int inverse, cudaStream_t stream) {
  const int chunks = row_bytes / 16;
  const long long total = (long long)L * chunks;
  int dev = 0, sms = 148;
  if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  // about four CTAs per SM over the whole launch, split across the heads
  long long want = ((long long)4 * sms + batch_heads - 1) / batch_heads;
  const long long need = (total + kThreads - 1) / kThreads;
  const int gx = (int)(want < 1 ? 1 : (want < need ? want : need));
  permute_rows_kernel<<<dim3(gx, batch_heads), kThreads, 0, stream>>>(
      static_cast<const uint4*>(src), static_cast<uint4*>(dst), perm, L, chunks, perm_per_head, inverse, total);
  return cudaGetLastError();
}

}  // namespace pisa
