// Covariance-aware top-k routing and the query-block pairing order.
//
// "PISA: Piecewise Sparse Attention Is Wiser for Efficient Diffusion Transformers", §2 방법론,
// 공분산 인식 라우팅: the block selection score combines the attention score with the block
// covariance norm M_j = ||H_j - Hbar||; blocks of high relevance or high heterogeneity are computed
// exactly, smoother ones are left to the Taylor terms.  Per query block i (fp32 throughout, so that
// near-ties resolve like the fp64 definition up to ~1e-6 relative):
//   s_ij = scale * qbar_i . kbar_j
//   P_ij = cnt_j exp(s_ij - max_l s_il) / sum_l cnt_l exp(s_il - max_l s_il)
//   r_ij = P_ij + lambda * M_j / sum_l M_l
//   S_i  = keep_k largest r_ij, ties to the lower j, written in ascending j.
// Top-k is an exact radix select on the IEEE bit patterns of r (r >= 0, so bit order is value
// order) followed by an ordered warp compaction; no sort is needed.
#include "route_body.cuh"

namespace pisa {
namespace {

template <int D, int kRows, int kCols>
__global__ void __launch_bounds__(kRouteThreads, 2) route_kernel(const float* __restrict__ qbar, const float* __restrict__ kbar,
                                                              const float* __restrict__ M, int L, int block, int nb,
                                                              float scale, int keep_k, float lam,
                                                              int32_t* __restrict__ sel, float* __restrict__ scores) {
  extern __shared__ __align__(16) float smem[];
  const int i0 = blockIdx.x * kRows;
  route_rows<D, kRows, kCols>(qbar, kbar, M, L, block, nb, scale, keep_k, lam, sel, scores, blockIdx.y, i0,
                       min(kRows, nb - i0), smem);
}

__global__ void __launch_bounds__(kRouteThreads) pair_kernel(const int32_t* __restrict__ sel, int nb, int keep_k,
                                                             int32_t* __restrict__ order) {
  extern __shared__ uint32_t psm[];
  pair_segment(sel, nb, keep_k, order, blockIdx.y, blockIdx.x, psm);
}

__global__ void identity_order(int nb, int32_t* __restrict__ order) {
  const int bh = blockIdx.y;
  for (int i = blockIdx.x * blockDim.x + threadIdx.x; i < nb; i += gridDim.x * blockDim.x)
    order[(size_t)bh * nb + i] = i;
}

template <int D, int kRows, int kCols>
cudaError_t launch_route_kernel(const Dims& g, const pisa_stats& st, int keep_k, float lam, int32_t* sel,
                                float* scores, cudaStream_t stream) {
  const size_t smem = route_smem_floats<D, kRows, kCols>(g.nb) * sizeof(float);
  cudaError_t e;
  if ((e = set_max_dynamic_smem(reinterpret_cast<const void*>(route_kernel<D, kRows, kCols>), smem)))
    return e;
  // lambda == 0 drops the M term: M is not read (it may be unwritten)
  route_kernel<D, kRows, kCols><<<dim3((g.nb + kRows - 1) / kRows, g.BH()), kRouteThreads, smem, stream>>>(
      st.qbar, st.kbar, lam > 0.f ? st.M : nullptr, g.L, g.block, g.nb, g.scale, keep_k, lam, sel, scores);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_route(const Dims& g, const pisa_stats& st, int keep_k, float lam, int32_t* sel,
                         int32_t* order, float* scores, cudaStream_t stream) {
  cudaError_t e;
  // 16 query blocks per CTA while their score rows fit comfortably in shared memory, else 8; one or
  // two centroids per thread (route_cols)
  const bool two = route_cols(g.nb) == 2;
  if (g.d == 64)   // (head_dim 64: one centroid per thread up to nb = 2048, which fits its registers)
    e = g.nb > 2048 ? launch_route_kernel<64, 8, 2>(g, st, keep_k, lam, sel, scores, stream)
                    : launch_route_kernel<64, 16, 1>(g, st, keep_k, lam, sel, scores, stream);
  else
    e = g.nb > 2048 ? launch_route_kernel<128, 8, 2>(g, st, keep_k, lam, sel, scores, stream)
        : two       ? launch_route_kernel<128, 16, 2>(g, st, keep_k, lam, sel, scores, stream)
                    : launch_route_kernel<128, 16, 1>(g, st, keep_k, lam, sel, scores, stream);
  if (e != cudaSuccess) return e;
  if (order) {
    if (g.block == 64 && keep_k > 0 && g.nb > 2) {
      const size_t psmem = pair_smem_bytes(g.nb);
      if ((e = set_max_dynamic_smem(reinterpret_cast<const void*>(pair_kernel), psmem))) return e;
      pair_kernel<<<dim3((g.nb + kSeg - 1) / kSeg, g.BH()), kRouteThreads, psmem, stream>>>(sel, g.nb, keep_k, order);
    } else {
      identity_order<<<dim3((g.nb + 255) / 256, g.BH()), 256, 0, stream>>>(g.nb, order);
    }
    if ((e = cudaGetLastError())) return e;
  }
  return cudaSuccess;
}

}  // namespace pisa
