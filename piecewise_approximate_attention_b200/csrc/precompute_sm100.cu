// Block statistics on sm_100a for bf16 inputs: TMA tiles, tcgen05 contractions for H_j.
//
// "PISA: Piecewise Sparse Attention Is Wiser for Efficient Diffusion Transformers", §2 방법론:
// the pre-computation step (하드웨어 구현 step 1) produces block centroids kbar_j and value sums
// (zeroth-order term), the global statistic Hbar = mean_j H_j with H_j = sum_n (k_n - kbar_j)^T v_n
// (first-order correction) and, for covariance-aware routing (공분산 인식 라우팅),
// M_j = ||H_j - Hbar||_F.  Query-block means qbar_i are produced in the same pass for routing.
//
// Both passes work on groups of kBlocksPerPart key blocks of one head and run persistently: one CTA
// per SM takes a contiguous range of groups and streams their tiles without a break, so the
// pipeline fills once per CTA and each group's epilogue overlaps the next group's loads (a CTA per
// group spent ~15% of its time filling and draining its own pipeline).
// Pass A streams 128-row tiles of Q, K, V with TMA, forms block column sums on the tensor core
// (against a block-indicator matrix), and accumulates sum_n k_n v_n^T over each group in TMEM with
// tcgen05 (both operands MN-major, fp32 accumulate; two TMEM buffers).  Its epilogue subtracts
// sum_j kbar_j vsum_j^T, giving the group's partial sum_j H_j.  The fixed-order reduction of the
// partials (hbar_reduce) gives Hbar.  Pass A also reduces max |v| per group; hbar_reduce turns it
// into the head's value scale (a power of two).  Pass B re-streams K, V, recomputes each H_j with
// one MMA chain per block into double-buffered TMEM and reduces ||H_j - kbar_j vsum_j^T - Hbar||^2
// in the epilogue, and writes the attention's fp16 value operands v / vscale and vsum / vscale from
// the tiles it streams.  Re-reading K, V (2 L d bf16) costs less HBM traffic than storing and
// re-reading H_j (nb d^2 fp32).
#include <algorithm>

#include "precompute_sm100.cuh"

namespace pisa {
namespace {
using namespace sm100;

// This CTA's contiguous share [u0, u1) of n groups (head-major, so a CTA's groups mostly belong to
// one head).
__device__ __forceinline__ void cta_groups(int n, int& u0, int& u1) {
  u0 = (int)((long long)n * blockIdx.x / gridDim.x);
  u1 = (int)((long long)n * (blockIdx.x + 1) / gridDim.x);
}

template <bool kFirstOrder>
__global__ void __launch_bounds__(kThreads, 1) stats_a_sm100(const __grid_constant__ KVMaps maps, const PreParams p,
                                                              int ngroups, int nbh) {
  extern __shared__ uint8_t smem_raw[];
  SmemA& sm = *reinterpret_cast<SmemA*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int warp = threadIdx.x >> 5;
  griddep_launch_dependents();      // the Hbar reduction may be scheduled now (it waits for this grid)
  if (warp == 5) {
    tmem_alloc(&sm.tmem_base, pass_a_tmem_cols(kFirstOrder));
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = sm.tmem_base;
  int u0, u1;
  cta_groups(ngroups * nbh, u0, u1);
  stats_a_body<kFirstOrder>(maps, p, sm, tmem, u0, u1, ngroups);
  if (warp == 5) {
    __syncwarp();
    tmem_dealloc(tmem, pass_a_tmem_cols(kFirstOrder));
  }
}

template <bool kDiff>
__global__ void __launch_bounds__(kThreads, 1) cov_norm_sm100(const __grid_constant__ KVMaps maps, const PreParams p,
                                                               int ngroups, int nbh) {
  extern __shared__ uint8_t smem_raw[];
  SmemB& sm = *reinterpret_cast<SmemB*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int warp = threadIdx.x >> 5;
  if (warp == 5) {
    tmem_alloc(&sm.tmem_base, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = sm.tmem_base;
  int u0, u1;
  cta_groups(ngroups * nbh, u0, u1);
  cov_norm_body<kDiff>(maps, p, sm, tmem, u0, u1, ngroups);
  if (warp == 5) {
    __syncwarp();
    tmem_dealloc(tmem, 512);
  }
}

// Zeroth-order pre-computation, second launch: one CTA per (head, group of kBlocksPerPart key
// blocks).  Every CTA of a head derives the head's value scale from the groups' max |v| (the same
// rule as hbar_reduce: the smallest power of two >= max|v| / 256); the first writes it.  Each CTA
// writes its blocks' fp16 value sums vsum / vscale and, when the scale is not 1, rewrites its rows
// of the fp16 value operand (stats_a_sm100<false> wrote them with scale 1).
__global__ void __launch_bounds__(256) value_scale_finish(const __nv_bfloat16* __restrict__ v, const PreParams p) {
  const int part = blockIdx.x, bh = blockIdx.y, nparts = gridDim.x;
  float mx = 0.f;
  for (int i = 0; i < nparts; ++i) mx = fmaxf(mx, p.vmax[(size_t)bh * nparts + i]);
  float sc = 1.f;
  while (mx > 256.f * sc && sc < 0x1p100f) sc *= 2.f;
  if (part == 0 && threadIdx.x == 0) p.st.vscale[bh] = sc;
  const float vinv = 1.f / sc;
  const int jb0 = part * kBlocksPerPart, jb1 = min(p.nb, jb0 + kBlocksPerPart);
  __half* vsop = reinterpret_cast<__half*>(p.st.vsum_op);
  for (int e = threadIdx.x; e < (jb1 - jb0) * D; e += blockDim.x) {
    const size_t so = ((size_t)bh * p.nb + jb0) * D + e;
    vsop[so] = __float2half_rn(p.st.vsum[so] * vinv);
  }
  if (sc == 1.f) return;
  const int row0 = jb0 * p.block, row1 = min(p.L, jb1 * p.block);
  const uint4* src = reinterpret_cast<const uint4*>(v + (size_t)bh * p.L * D);
  uint4* dst = reinterpret_cast<uint4*>(reinterpret_cast<__half*>(p.st.v_op) + (size_t)bh * p.L * D);
  for (size_t e = (size_t)row0 * (D / 8) + threadIdx.x; e < (size_t)row1 * (D / 8); e += blockDim.x) {
    const uint4 u = src[e];
    const uint32_t w[4] = {u.x, u.y, u.z, u.w};
    uint32_t hw[4];
#pragma unroll
    for (int x = 0; x < 4; ++x) {
      const __half2 h2 = __floats2half2_rn(__uint_as_float(w[x] << 16) * vinv, __uint_as_float(w[x] & 0xffff0000u) * vinv);
      hw[x] = *reinterpret_cast<const uint32_t*>(&h2);
    }
    dst[e] = make_uint4(hw[0], hw[1], hw[2], hw[3]);
  }
}

}  // namespace

cudaError_t launch_precompute_sm100(const Dims& g, const void* q, const void* k, const void* v, const pisa_stats& st,
                                    void* ws, bool first_order, unsigned long long wait_ns, int fault,
                                    cudaStream_t stream) {
  KVMaps maps;
  const uint64_t bh = (uint64_t)g.BH();
  if (!encode_bf16_3d(&maps.q, q, D, g.L, bh, 128) || !encode_bf16_3d(&maps.k, k, D, g.L, bh, 128) ||
      !encode_bf16_3d(&maps.v, v, D, g.L, bh, 128))
    return cudaErrorInvalidValue;
  PreParams p;
  p.L = g.L;
  p.nb = g.nb;
  p.block = g.block;
  p.scale = g.scale;
  p.st = st;
  p.partials = reinterpret_cast<float*>(static_cast<char*>(ws) + kStatusBytes);
  p.vmax = reinterpret_cast<float*>(static_cast<char*>(ws) + vmax_offset(g));
  p.status = static_cast<int*>(ws);
  p.wait_ns = wait_ns;
  p.fault = fault;
  const size_t smem_a = sizeof(SmemA) + 1024, smem_b = sizeof(SmemB) + 1024;
  cudaError_t e;
  if ((e = set_max_dynamic_smem(reinterpret_cast<const void*>(stats_a_sm100<true>), smem_a))) return e;
  if ((e = set_max_dynamic_smem(reinterpret_cast<const void*>(stats_a_sm100<false>), smem_a))) return e;
  if ((e = set_max_dynamic_smem(reinterpret_cast<const void*>(cov_norm_sm100<false>), smem_b))) return e;
  if ((e = set_max_dynamic_smem(reinterpret_cast<const void*>(cov_norm_sm100<true>), smem_b))) return e;
  const int nparts = num_parts(g), nbh = g.BH();
  // persistent grids: one CTA per SM (each needs most of an SM's shared memory), at most one per group
  int nsm = 0;
  if ((e = sm_count(&nsm))) return e;
  const int ctas = std::min(nparts * nbh, nsm);
  if (!first_order) {
    // one group per CTA: this pass (three tiles read, one written per tile, no group epilogue) runs
    // at the copy bandwidth with a CTA per group and measured ~2.5% slower persistent
    stats_a_sm100<false><<<nparts * nbh, kThreads, smem_a, stream>>>(maps, p, nparts, nbh);
    value_scale_finish<<<dim3(nparts, g.BH()), 256, 0, stream>>>(static_cast<const __nv_bfloat16*>(v), p);
    return cudaGetLastError();
  }
  // The reduction and pass B are programmatic dependents: pass B's CTAs take the SMs that pass A
  // leaves and start streaming K and V (which nothing here writes) while the last pass-A CTAs and
  // the reduction finish; its epilogue waits for them before it reads their results.
  stats_a_sm100<true><<<ctas, kThreads, smem_a, stream>>>(maps, p, nparts, nbh);
  if ((e = cudaGetLastError())) return e;
  if ((e = launch_hbar_reduce(g, p.partials, nparts, p.vmax, st, stream, true))) return e;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(ctas);
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = smem_b;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  if (st.hdiff_op) return cudaLaunchKernelEx(&cfg, cov_norm_sm100<true>, maps, p, nparts, nbh);
  return cudaLaunchKernelEx(&cfg, cov_norm_sm100<false>, maps, p, nparts, nbh);
}

}  // namespace pisa
