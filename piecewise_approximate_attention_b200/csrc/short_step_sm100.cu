// Pre-computation and routing of short sequences in one launch: one thread-block cluster per head.
//
// "PISA: Piecewise Sparse Attention Is Wiser for Efficient Diffusion Transformers": §1 문제 정의
// and §4 실험 결과 stress that sparse attention must keep its edge at short sequences (4K tokens),
// where the fixed cost of the pre-computation (§2 하드웨어 구현 step 1) and of the routing
// (공분산 인식 라우팅) weighs most.  Launched as separate kernels, pass A, the Hbar reduction,
// pass B, the router and the pairing each pay a launch, a ramp-up and a tail.  Here they run in one
// kernel: the cluster of CTAs of a head (one CTA per group of kBlocksPerPart key blocks, at most 8,
// so nb <= 128) meets at hardware cluster barriers between the phases.  The groups' partial sums
// of H_j go through the workspace in L2: reading them from the other CTAs' shared memory (DSMEM)
// measured ~9.5 us for the reduction at 4.6K tokens, several times the L2 round trip.
//
//   1. pass A (stats_a_body): block sums, max |v|, the group's partial sum of H_j -> workspace
//   2. Hbar = (sum of the partials, in group order) / nb, split by elements over the cluster's CTAs;
//      the value scale from the groups' max |v|
//   3. pass B (cov_norm_body): M_j, the fp16 value operands (and H_j / s (H_j - Hbar) on request)
//   4. routing of the CTA's own 16 query blocks (route_rows)
//   5. the pairing order of the head's query blocks (pair_segment, rank 0)
//
// Every phase uses the same code, groups and summation orders as the separate kernels, so the
// statistics, selections, scores and order are bit-identical to pisa_precompute + pisa_route.
// Every CTA reaches every cluster barrier: the bodies' bounded waits return (after recording a
// timeout in the status word) instead of leaving a CTA behind.
#include <mutex>

#include "precompute_sm100.cuh"
#include "route_body.cuh"

namespace pisa {
namespace {
using namespace sm100;

constexpr int kShortThreads = 256;   // 8 warps: the routing body's CTA size; passes A/B use warps 0-5
constexpr int kMaxCluster = 8;       // portable cluster size: nb <= 8 * kBlocksPerPart = 128

static_assert(kShortThreads == kRouteThreads, "the routing body runs on the whole CTA");

struct ShortParams {
  PreParams pre;
  int keep_k;
  float lam;
  int32_t* sel;
  int32_t* order;
  float* scores;
};

__device__ __forceinline__ uint32_t cluster_rank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}

// All threads of every CTA of the cluster.  Global-memory writes made before it by any thread of
// the cluster are visible to every thread of the cluster after it (gpu-scope fences on both sides,
// for data that the other CTAs then read with ordinary loads).
__device__ __forceinline__ void cluster_sync_all() {
  __threadfence();
  asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
  __threadfence();
}

__device__ __forceinline__ void mbar_inval(uint64_t* bar) {
  asm volatile("mbarrier.inval.shared::cta.b64 [%0];" ::"r"(smem_u32(bar)) : "memory");
}

// The shared memory of one CTA, reused phase by phase (cluster barriers separate the phases).
union alignas(1024) ShortSmem {
  SmemA a;                                    // phase 1
  SmemB b;                                    // phase 3
  float route[route_smem_floats<D, 16, 1>(128)];                                              // phase 4
  uint32_t pair[pair_smem_bytes(128) / 4];                                                 // phase 5
};
static_assert(sizeof(ShortSmem::route) / 4 >= route_smem_floats<D, 16, 1>(128), "routing scratch");

template <bool kDiff>
__global__ void __launch_bounds__(kShortThreads, 1) short_step_sm100(const __grid_constant__ KVMaps maps,
                                                                     const ShortParams sp) {
  extern __shared__ uint8_t smem_raw[];
  ShortSmem& sm = *reinterpret_cast<ShortSmem*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const PreParams& p = sp.pre;
  const int warp = threadIdx.x >> 5;
  const int nparts = gridDim.x;                      // == cluster size: one cluster per head
  const int rank = (int)cluster_rank();
  const int bh = blockIdx.y;
  __shared__ uint32_t tmem_base;

  if (warp == 5) {
    tmem_alloc(&tmem_base, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = tmem_base;

  // ---- 1. pass A of this CTA's group ----
  const int unit = bh * nparts + rank;                // group `rank` of head bh
  stats_a_body<true>(maps, p, sm.a, tmem, unit, unit + 1, nparts);
  if (threadIdx.x == 0) {
    for (int s = 0; s < 2; ++s) {
      mbar_inval(&sm.a.full[s]);
      mbar_inval(&sm.a.empty[s]);
      mbar_inval(&sm.a.sums_full[s]);
      mbar_inval(&sm.a.sums_empty[s]);
      mbar_inval(&sm.a.acc_full[s]);
      mbar_inval(&sm.a.acc_empty[s]);
    }
    mbar_inval(&sm.a.drain);
  }
  cluster_sync_all();

  // ---- 2. Hbar: element float4 f of the head is reduced by CTA f % nparts, over the groups in order
  {
    const float nbf = (float)p.nb;
    float* hbar = p.st.hbar + (size_t)bh * D * D;
    __nv_bfloat16* hop = static_cast<__nv_bfloat16*>(p.st.hbar_op) + (size_t)bh * D * D;
    constexpr int kG = 4;                              // float4 elements per thread in flight at once
    const int stride = nparts * kShortThreads;
    for (int f0 = rank + nparts * threadIdx.x; f0 < D * D / 4; f0 += kG * stride) {
      // every group's float4 of kG elements first (all loads in flight together, from L2: the
      // other CTAs wrote them), then the sums in group order
      const float4* part = reinterpret_cast<const float4*>(p.partials + (size_t)bh * nparts * D * D);
      float4 v[kG][kMaxCluster];
#pragma unroll
      for (int g = 0; g < kG; ++g) {
        const int f = f0 + g * stride;
#pragma unroll
        for (int i = 0; i < kMaxCluster; ++i)
          if (f < D * D / 4 && i < nparts) v[g][i] = __ldcg(part + (size_t)i * (D * D / 4) + f);
      }
#pragma unroll
      for (int g = 0; g < kG; ++g) {
        const int f = f0 + g * stride;
        if (f >= D * D / 4) break;
        float4 s = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
        for (int i = 0; i < kMaxCluster; ++i) {
          if (i < nparts) {
            s.x += v[g][i].x;
            s.y += v[g][i].y;
            s.z += v[g][i].z;
            s.w += v[g][i].w;
          }
        }
        const float h[4] = {s.x / nbf, s.y / nbf, s.z / nbf, s.w / nbf};
        *reinterpret_cast<float4*>(hbar + 4 * f) = make_float4(h[0], h[1], h[2], h[3]);
        const int a = (4 * f) / D, c0 = (4 * f) % D;
#pragma unroll
        for (int x = 0; x < 4; ++x) hop[(size_t)(c0 + x) * D + a] = __float2bfloat16_rn(p.scale * h[x]);
      }
    }
    if (rank == 0 && threadIdx.x == 0) {
      float mx = 0.f;
      for (int i = 0; i < nparts; ++i) mx = fmaxf(mx, p.vmax[(size_t)bh * nparts + i]);
      float sc = 1.f;
      while (mx > 256.f * sc && sc < 0x1p100f) sc *= 2.f;
      p.st.vscale[bh] = sc;
    }
  }
  cluster_sync_all();      // Hbar and the value scale written

  // ---- 3. pass B of this CTA's group ----
  cov_norm_body<kDiff>(maps, p, sm.b, tmem, unit, unit + 1, nparts);
  if (threadIdx.x == 0) {
    for (int s = 0; s < kStagesB; ++s) {
      mbar_inval(&sm.b.full[s]);
      mbar_inval(&sm.b.empty[s]);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_inval(&sm.b.acc_full[b]);
      mbar_inval(&sm.b.acc_empty[b]);
    }
    mbar_inval(&sm.b.drain);
  }
  cluster_sync_all();      // every M_j and centroid of the head written

  // ---- 4. routing of query blocks [16 rank, 16 rank + 16) ----
  {
    const int i0 = rank * kBlocksPerPart;
    route_rows<D, kBlocksPerPart, 1>(p.st.qbar, p.st.kbar, sp.lam > 0.f ? p.st.M : nullptr, p.L, p.block, p.nb, p.scale,
                                  sp.keep_k, sp.lam, sp.sel, sp.scores, bh, i0, min(kBlocksPerPart, p.nb - i0),
                                  sm.route);
  }
  cluster_sync_all();      // every selection of the head written

  // ---- 5. the pairing order (block 64), or the identity ----
  if (sp.order && rank == 0) {
    if (p.block == 64 && sp.keep_k > 0 && p.nb > 2) {
      pair_segment(sp.sel, p.nb, sp.keep_k, sp.order, bh, 0, sm.pair);
    } else {
      for (int i = threadIdx.x; i < p.nb; i += kShortThreads) sp.order[(size_t)bh * p.nb + i] = i;
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 5) {
    __syncwarp();
    tmem_dealloc(tmem, 512);
  }
}

size_t short_smem_bytes() { return sizeof(ShortSmem) + 1024; }

// Whether a cluster of `nparts` CTAs of this kernel fits on the current device (asked once per
// device, variant and cluster size, so that calls made under stream capture do not repeat the query).
std::mutex g_fit_mu;
signed char g_fit[64][2][kMaxCluster + 1];   // 0 unknown, -1 none fits, else clusters co-resident

template <bool kDiff>
cudaError_t launch_short(const KVMaps& maps, const ShortParams& sp, int nparts, int bh, cudaStream_t stream,
                         bool* launched) {
  const size_t smem = short_smem_bytes();
  cudaError_t e = set_max_dynamic_smem(reinterpret_cast<const void*>(short_step_sm100<kDiff>), smem);
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(nparts, bh, 1);
  cfg.blockDim = dim3(kShortThreads, 1, 1);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = nparts;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  // a cluster of this size and shared memory must fit on the device; otherwise the caller runs the
  // separate kernels
  int dev = 0;
  if ((e = cudaGetDevice(&dev)) != cudaSuccess) return e;
  signed char fit = 0;
  if (dev >= 0 && dev < 64 && nparts <= kMaxCluster) {
    std::lock_guard<std::mutex> lock(g_fit_mu);
    fit = g_fit[dev][kDiff ? 1 : 0][nparts];
    if (fit == 0) {
      int clusters = 0;
      const cudaError_t q = cudaOccupancyMaxActiveClusters(&clusters, short_step_sm100<kDiff>, &cfg);
      if (q != cudaSuccess) (void)cudaGetLastError();
      fit = q == cudaSuccess ? (signed char)(clusters > 127 ? 127 : clusters) : -1;
      if (fit == 0) fit = -1;
      g_fit[dev][kDiff ? 1 : 0][nparts] = fit;
    }
  }
  // one cluster per head, all co-resident: with more heads than clusters fit, the separate kernels
  // (which need no co-residency) are faster than a second wave of clusters
  if (fit < 1 || bh > fit) {
    *launched = false;
    return cudaSuccess;
  }
  e = cudaLaunchKernelEx(&cfg, short_step_sm100<kDiff>, maps, sp);
  *launched = e == cudaSuccess;
  return e;
}

}  // namespace

bool short_step_eligible(const Dims& g) {
  return g.d == D && bf16_inputs(g.dtype) && g.nb <= kMaxCluster * kBlocksPerPart;
}

cudaError_t launch_short_step_sm100(const Dims& g, const void* q, const void* k, const void* v, const pisa_stats& st,
                                    void* ws, int keep_k, float lam, int32_t* sel, int32_t* order, float* scores,
                                    cudaStream_t stream, bool* launched) {
  *launched = false;
  if (!short_step_eligible(g)) return cudaSuccess;
  KVMaps maps;
  const uint64_t bh = (uint64_t)g.BH();
  if (!encode_bf16_3d(&maps.q, q, D, g.L, bh, 128) || !encode_bf16_3d(&maps.k, k, D, g.L, bh, 128) ||
      !encode_bf16_3d(&maps.v, v, D, g.L, bh, 128))
    return cudaErrorInvalidValue;
  ShortParams sp;
  sp.pre.L = g.L;
  sp.pre.nb = g.nb;
  sp.pre.block = g.block;
  sp.pre.scale = g.scale;
  sp.pre.st = st;
  sp.pre.partials = reinterpret_cast<float*>(static_cast<char*>(ws) + kStatusBytes);
  sp.pre.vmax = reinterpret_cast<float*>(static_cast<char*>(ws) + vmax_offset(g));
  sp.pre.status = static_cast<int*>(ws);
  sp.pre.wait_ns = kWaitLimitNs;
  sp.keep_k = keep_k;
  sp.lam = lam;
  sp.sel = sel;
  sp.order = order;
  sp.scores = scores;
  const int nparts = num_parts(g);
  return st.hdiff_op ? launch_short<true>(maps, sp, nparts, g.BH(), stream, launched)
                     : launch_short<false>(maps, sp, nparts, g.BH(), stream, launched);
}

}  // namespace pisa
