// Token reordering before blocking (PAROAttention, "Pattern-Aware ReOrdering", abstract): rows of
// a [B*H][L][row_bytes] tensor are gathered through a permutation (dst[i] = src[perm[i]]) or
// scattered back with its inverse (dst[perm[i]] = src[i]), so that the blocks PISA forms over the
// reordered sequence follow another axis order of the video's (frames, height, width) grid.
//
// HBM-bound copy: every row is read once and written once as 16-byte vectors; consecutive threads
// take consecutive 16-byte chunks of a row, so each warp moves whole rows with full sectors.
// The grid is sized to a few CTAs per SM and strides over the rows; a row of 8, 16 or 32 chunks is
// indexed with shifts, and indices are 32-bit unless a head holds more than 2^31 chunks.
#include "common.cuh"

namespace pisa {
namespace {

constexpr int kThreads = 256;
constexpr int kUnroll = 4;

// kShift >= 0: a row is 2^kShift chunks (row index and chunk by shifts); -1: any count (divisions).
// Idx: 32-bit indices when a head's chunk count leaves room for the strided loop, else 64-bit.
template <int kShift, typename Idx>
__global__ void __launch_bounds__(kThreads) permute_rows_kernel(const uint4* __restrict__ src, uint4* __restrict__ dst,
                                                                const int32_t* __restrict__ perm, int L,
                                                                int chunks, int perm_per_head, int inverse, Idx total) {
  const int bh = blockIdx.y;
  const int32_t* pr = perm + (perm_per_head ? (size_t)bh * L : 0);
  const size_t base = (size_t)bh * L * chunks;
  const Idx stride = (Idx)gridDim.x * kThreads;
  // kUnroll chunks per thread per round: all loads are issued before the stores
  for (Idx e0 = (Idx)blockIdx.x * kThreads + threadIdx.x; e0 < total; e0 += kUnroll * stride) {
    uint4 val[kUnroll];
    Idx to[kUnroll];
#pragma unroll
    for (int u = 0; u < kUnroll; ++u) {
      const Idx e = e0 + u * stride;
      to[u] = -1;
      if (e < total) {
        const Idx i = kShift >= 0 ? e >> kShift : e / chunks;
        const Idx c = kShift >= 0 ? e & ((1 << kShift) - 1) : e - i * chunks;
        const int j = pr[i];
        if (j >= 0 && j < L) {   // out-of-range entries are skipped (documented in pisa.h)
          const Idx from = inverse ? i : (Idx)j;
          to[u] = (inverse ? (Idx)j : i) * chunks + c;
          val[u] = src[base + (size_t)from * chunks + c];
        }
      }
    }
#pragma unroll
    for (int u = 0; u < kUnroll; ++u)
      if (to[u] >= 0) dst[base + (size_t)to[u]] = val[u];
  }
}

template <typename Idx>
void launch_idx(const uint4* s4, uint4* d4, const int32_t* perm, int L, int chunks, int per_head, int inverse,
                Idx total, dim3 grid, cudaStream_t stream) {
  if (chunks == 16)
    permute_rows_kernel<4, Idx><<<grid, kThreads, 0, stream>>>(s4, d4, perm, L, chunks, per_head, inverse, total);
  else if (chunks == 32)
    permute_rows_kernel<5, Idx><<<grid, kThreads, 0, stream>>>(s4, d4, perm, L, chunks, per_head, inverse, total);
  else if (chunks == 8)
    permute_rows_kernel<3, Idx><<<grid, kThreads, 0, stream>>>(s4, d4, perm, L, chunks, per_head, inverse, total);
  else
    permute_rows_kernel<-1, Idx><<<grid, kThreads, 0, stream>>>(s4, d4, perm, L, chunks, per_head, inverse, total);
}

}  // namespace

cudaError_t launch_permute_rows(const void* src, void* dst, const int32_t* perm, int batch_heads, int L,
                                int row_bytes, int perm_per_head, int inverse, cudaStream_t stream) {
  const int chunks = row_bytes / 16;
  const long long total = (long long)L * chunks;
  int sms = 148;
  sm_count(&sms);
  // about four CTAs per SM over the whole launch, split across the heads
  long long want = ((long long)4 * sms + batch_heads - 1) / batch_heads;
  const long long need = (total + kThreads - 1) / kThreads;
  const int gx = (int)(want < 1 ? 1 : (want < need ? want : need));
  const dim3 grid(gx, batch_heads);
  const uint4* s4 = static_cast<const uint4*>(src);
  uint4* d4 = static_cast<uint4*>(dst);
  // the strided loop may step past total by kUnroll grid strides before it stops
  const long long slack = (long long)kUnroll * gx * kThreads;
  if (total + slack < 0x7fffffffLL)
    launch_idx<int>(s4, d4, perm, L, chunks, perm_per_head, inverse, (int)total, grid, stream);
  else
    launch_idx<long long>(s4, d4, perm, L, chunks, perm_per_head, inverse, total, grid, stream);
  return cudaGetLastError();
}

}  // namespace pisa
