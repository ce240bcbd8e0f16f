// Block statistics on sm_100a for bf16 inputs: TMA tiles, tcgen05 contractions for H_j.
//
// "PISA: Piecewise Sparse Attention Is Wiser for Efficient Diffusion Transformers", §2 방법론:
// the pre-computation step (하드웨어 구현 step 1) produces block centroids kbar_j and value sums
// (zeroth-order term), the global statistic Hbar = mean_j H_j with H_j = sum_n (k_n - kbar_j)^T v_n
// (first-order correction) and, for covariance-aware routing (공분산 인식 라우팅),
// M_j = ||H_j - Hbar||_F.  Query-block means qbar_i are produced in the same pass for routing.
//
// Pass A (one CTA per head and group of kBlocksPerPart key blocks): streams 128-row tiles of Q, K, V
// with TMA, reduces block column sums on CUDA cores straight from the swizzled tiles, and
// accumulates sum_n k_n v_n^T over the whole group in TMEM with tcgen05 (both operands MN-major,
// fp32 accumulate).  Its epilogue subtracts sum_j kbar_j vsum_j^T, giving the group's partial
// sum_j H_j.  The fixed-order reduction of the partials (hbar_reduce) gives Hbar.
// Pass A also reduces max |v| per group; hbar_reduce turns it into the head's value scale (a power
// of two).  Pass B (one CTA per head and group of key blocks): re-streams K, V, recomputes each H_j
// with one MMA chain per block into double-buffered TMEM and reduces ||H_j - kbar_j vsum_j^T -
// Hbar||^2 in the epilogue, and writes the attention's fp16 value operands v / vscale and
// vsum / vscale from the tiles it streams.  Re-reading K, V (2 L d bf16) costs less HBM traffic than storing and re-reading
// H_j (nb d^2 fp32).
#include <cuda_fp16.h>

#include "common.cuh"
#include "sm100.cuh"

namespace pisa {
namespace {
using namespace sm100;

constexpr int D = 128;
constexpr int kThreads = 192;
constexpr int kHalf = 128 * 64 * 2;      // 128 rows x 64 columns of bf16: 16 KB
constexpr int kTile = 2 * kHalf;         // 128 x 128 bf16 tile: 32 KB
constexpr uint32_t kIdescKV = idesc_bf16_f32(128, 128, true, true);   // D[a][c] += sum_n K[n][a] V[n][c]

__device__ __forceinline__ void bar_epi() { asm volatile("bar.sync 1, 128;" ::: "memory"); }

// Every epilogue thread reaches this after a bounded wait; the OR-reduction at the barrier gives all 128
// threads the same answer, so no later named barrier can strand a warp.
__device__ __forceinline__ bool epi_any_failed(bool failed) {
  uint32_t r;
  asm volatile(
      "{\n\t.reg .pred pi, po;\n\t"
      "setp.ne.u32 pi, %1, 0;\n\t"
      "bar.red.or.pred po, 1, 128, pi;\n\t"
      "selp.u32 %0, 1, 0, po;\n\t}"
      : "=r"(r)
      : "r"((uint32_t)failed)
      : "memory");
  return r != 0;
}

__device__ __forceinline__ bool wait_bar(uint64_t* bar, uint32_t parity, int* abort, int* status,
                                         unsigned long long ns) {
  if (mbar_wait_bounded(bar, parity, abort, ns)) return true;
  *reinterpret_cast<volatile int*>(abort) = 1;
  set_status(status, PISA_DEVERR_WAIT_TIMEOUT);
  return false;
}

// Sums of 8 consecutive columns (chunk cc of 16) over the rows r in [r0, r1) with r = rg (mod 8), read
// from a 128B-swizzled [128 x 128] bf16 tile.  r0 is a multiple of 8.  amax (if given) tracks max |x|.
__device__ __forceinline__ void colsum8(const uint8_t* tile, int cc, int rg, int r0, int r1, float acc[8],
                                        float* amax = nullptr) {
  const uint8_t* base = tile + (cc >> 3) * kHalf + (((cc & 7) ^ rg) << 4);
#pragma unroll 4
  for (int r = r0 + rg; r < r1; r += 8) {
    const uint4 u = *reinterpret_cast<const uint4*>(base + r * 128);
    acc[0] += __uint_as_float(u.x << 16);
    acc[1] += __uint_as_float(u.x & 0xffff0000u);
    acc[2] += __uint_as_float(u.y << 16);
    acc[3] += __uint_as_float(u.y & 0xffff0000u);
    acc[4] += __uint_as_float(u.z << 16);
    acc[5] += __uint_as_float(u.z & 0xffff0000u);
    acc[6] += __uint_as_float(u.w << 16);
    acc[7] += __uint_as_float(u.w & 0xffff0000u);
    if (amax) {
      // |x| of two packed bf16 at once: clear both sign bits; the larger magnitude sets the max
      const uint32_t a0 = u.x & 0x7fff7fffu, a1 = u.y & 0x7fff7fffu, a2 = u.z & 0x7fff7fffu, a3 = u.w & 0x7fff7fffu;
      float m = *amax;
      m = fmaxf(m, fmaxf(__uint_as_float(a0 << 16), __uint_as_float(a0 & 0xffff0000u)));
      m = fmaxf(m, fmaxf(__uint_as_float(a1 << 16), __uint_as_float(a1 & 0xffff0000u)));
      m = fmaxf(m, fmaxf(__uint_as_float(a2 << 16), __uint_as_float(a2 & 0xffff0000u)));
      m = fmaxf(m, fmaxf(__uint_as_float(a3 << 16), __uint_as_float(a3 & 0xffff0000u)));
      *amax = m;
    }
  }
}

struct KVMaps {
  CUtensorMap q, k, v;     // [BH][L][128] bf16, box {64, 128, 1}
};

struct PreParams {
  int L, nb, block;
  float scale;               // softmax scale (folded into the per-block first-order operand copy)
  pisa_stats st;
  float* partials;
  float* vmax;               // [BH][nparts] max |v| per group (pass A)
  int* status;
  unsigned long long wait_ns;
};

// ----------------------------------------------------------------------------------------------
// Pass A
// ----------------------------------------------------------------------------------------------
struct alignas(1024) SmemA {
  uint8_t q[2][kTile];
  uint8_t k[2][kTile];
  uint8_t v[2][kTile];
  float red[3][4][128];
  float ck[2][128], cv[2][128];
  uint64_t full[2], empty[2], acc_done;
  uint32_t tmem_base;
  int abort;
};

// kFirstOrder: also accumulate the group's partial sum of H_j (tensor core) for Hbar.  Without it
// (the zeroth-order pre-computation) the CTA writes the fp16 value operand with scale 1 from the V
// tiles it streams, on the chance that the head's value scale is 1; value_scale_finish rewrites it
// when it is not.
template <bool kFirstOrder>
__global__ void __launch_bounds__(kThreads, 1) stats_a_sm100(const __grid_constant__ KVMaps maps, const PreParams p) {
  extern __shared__ uint8_t smem_raw[];
  SmemA& sm = *reinterpret_cast<SmemA*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int part = blockIdx.x, bh = blockIdx.y, nparts = gridDim.x;
  const int jb0 = part * kBlocksPerPart, jb1 = min(p.nb, jb0 + kBlocksPerPart);
  const int row0 = jb0 * p.block, row1 = min(p.L, jb1 * p.block);
  const int ntile = (row1 - row0 + 127) / 128;
  const int bpt = 128 / p.block;

  if (threadIdx.x == 0) {
    for (int s = 0; s < 2; ++s) {
      mbar_init(&sm.full[s], 1);
      mbar_init(&sm.empty[s], kFirstOrder ? 129 : 128);   // the 128 column-sum threads (+ the MMA commit)
    }
    mbar_init(&sm.acc_done, 1);
    sm.abort = 0;
    fence_mbar_init();
  }
  if (kFirstOrder && warp == 5) {
    tmem_alloc(&sm.tmem_base, 128);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = kFirstOrder ? sm.tmem_base : 0u;

  if (warp == 4) {
    if (lane == 0) {
      int issued = 0;
      bool ok = true;
      for (int t = 0; t < ntile; ++t) {
        const int s = t & 1;
        if (t >= 2 && !(ok = wait_bar(&sm.empty[s], ((t >> 1) - 1) & 1, &sm.abort, p.status, p.wait_ns))) break;
        const int y = row0 + t * 128;
        mbar_expect_tx(&sm.full[s], 3 * kTile);
        tma_load_3d(sm.q[s], &maps.q, &sm.full[s], 0, y, bh);
        tma_load_3d(sm.q[s] + kHalf, &maps.q, &sm.full[s], 64, y, bh);
        tma_load_3d(sm.k[s], &maps.k, &sm.full[s], 0, y, bh);
        tma_load_3d(sm.k[s] + kHalf, &maps.k, &sm.full[s], 64, y, bh);
        tma_load_3d(sm.v[s], &maps.v, &sm.full[s], 0, y, bh);
        tma_load_3d(sm.v[s] + kHalf, &maps.v, &sm.full[s], 64, y, bh);
        ++issued;
      }
      {   // let issued copies land before shared memory is released (normally already landed)
        for (int t = max(0, issued - 2); t < issued; ++t) mbar_drain(&sm.full[t & 1], (t >> 1) & 1, p.wait_ns);
      }
    }
  } else if (warp == 5) {
    if (kFirstOrder && lane == 0) {
      bool ok = true;
      for (int t = 0; t < ntile && ok; ++t) {
        const int s = t & 1;
        if (!(ok = wait_bar(&sm.full[s], (t >> 1) & 1, &sm.abort, p.status, p.wait_ns))) break;
        tc_fence_after();
        const uint32_t ka = smem_u32(sm.k[s]), va = smem_u32(sm.v[s]);
#pragma unroll
        for (int kk = 0; kk < 8; ++kk)
          mma_ss(tmem, smem_desc_sw128(ka + kk * 2048, kHalf, 1024), smem_desc_sw128(va + kk * 2048, kHalf, 1024),
                 kIdescKV, (t > 0 || kk > 0) ? 1u : 0u);
        mma_commit(&sm.empty[s]);
      }
      mma_commit(&sm.acc_done);
      const uint64_t t0 = globaltimer_ns();
      while (!mbar_try_wait(&sm.acc_done, 0) && globaltimer_ns() - t0 < p.wait_ns) {}
    }
  } else {
    // column sums + rank-1 centring terms (threads 0..127)
    const int tid = threadIdx.x, cc = tid & 15, rg = tid >> 4;
    float corr[kFirstOrder ? D : 1];
#pragma unroll
    for (int c = 0; c < (kFirstOrder ? D : 1); ++c) corr[c] = 0.f;
    bool ok = true;
    int nblk = 0;
    float vabs = 0.f;
    for (int t = 0; t < ntile; ++t) {
      const int s = t & 1;
      ok = !epi_any_failed(!wait_bar(&sm.full[s], (t >> 1) & 1, &sm.abort, p.status, p.wait_ns));
      if (!ok) break;
      for (int b = 0; b < bpt; ++b) {
        const int j = jb0 + t * bpt + b;
        if (j >= jb1) break;
        const int cnt = block_count(j, p.L, p.block);
        const int r0 = b * p.block;
        float aq[8] = {0, 0, 0, 0, 0, 0, 0, 0}, ak[8] = {0, 0, 0, 0, 0, 0, 0, 0}, av[8] = {0, 0, 0, 0, 0, 0, 0, 0};
        colsum8(sm.q[s], cc, rg, r0, r0 + cnt, aq);
        colsum8(sm.k[s], cc, rg, r0, r0 + cnt, ak);
        colsum8(sm.v[s], cc, rg, r0, r0 + cnt, av, &vabs);
        // lanes l and l ^ 16 hold the same 8 columns for row groups 2w and 2w + 1: add them in
        // registers, then one row of partial sums per warp goes through shared memory
#pragma unroll
        for (int x = 0; x < 8; ++x) {
          aq[x] += __shfl_xor_sync(0xffffffffu, aq[x], 16);
          ak[x] += __shfl_xor_sync(0xffffffffu, ak[x], 16);
          av[x] += __shfl_xor_sync(0xffffffffu, av[x], 16);
        }
        if (lane < 16) {
          float4* dq = reinterpret_cast<float4*>(&sm.red[0][warp][cc * 8]);
          float4* dk = reinterpret_cast<float4*>(&sm.red[1][warp][cc * 8]);
          float4* dv = reinterpret_cast<float4*>(&sm.red[2][warp][cc * 8]);
          dq[0] = make_float4(aq[0], aq[1], aq[2], aq[3]);
          dq[1] = make_float4(aq[4], aq[5], aq[6], aq[7]);
          dk[0] = make_float4(ak[0], ak[1], ak[2], ak[3]);
          dk[1] = make_float4(ak[4], ak[5], ak[6], ak[7]);
          dv[0] = make_float4(av[0], av[1], av[2], av[3]);
          dv[1] = make_float4(av[4], av[5], av[6], av[7]);
        }
        bar_epi();
        const int c = tid;
        float sq = 0.f, sk = 0.f, sv = 0.f;
#pragma unroll
        for (int g = 0; g < 4; ++g) {
          sq += sm.red[0][g][c];
          sk += sm.red[1][g][c];
          sv += sm.red[2][g][c];
        }
        const float inv = 1.f / (float)cnt;
        const size_t so = ((size_t)bh * p.nb + j) * D + c;
        p.st.qbar[so] = sq * inv;
        p.st.kbar[so] = sk * inv;
        p.st.vsum[so] = sv;
        reinterpret_cast<__nv_bfloat16*>(p.st.kbar_op)[so] = __float2bfloat16_rn(sk * inv);
        if constexpr (kFirstOrder) {
          const int pb = nblk & 1;
          sm.ck[pb][c] = sk * inv;
          sm.cv[pb][c] = sv;
          bar_epi();     // also: every thread has read red[] before the next block writes it
          const float ka = sm.ck[pb][tid];
#pragma unroll
          for (int x = 0; x < D; ++x) corr[x] = fmaf(ka, sm.cv[pb][x], corr[x]);
        } else {
          bar_epi();     // every thread has read red[] before the next block writes it
        }
        ++nblk;
      }
      if constexpr (!kFirstOrder) {
        // fp16 value operand with scale 1 (exact for every bf16 value in fp16's range): 16-byte
        // chunks of the swizzled V tile, consecutive chunks per thread
        __half* vop = reinterpret_cast<__half*>(p.st.v_op) + (size_t)bh * p.L * D;
        const int rbase = row0 + t * 128;
        for (int q = tid; q < 128 * 16; q += 128) {
          const int row = q >> 4, c = q & 15;
          if (rbase + row >= row1) break;
          const uint4 u = *reinterpret_cast<const uint4*>(sm.v[s] + (c >> 3) * kHalf + row * 128 + (((c & 7) ^ (row & 7)) << 4));
          const uint32_t w[4] = {u.x, u.y, u.z, u.w};
          uint32_t hw[4];
#pragma unroll
          for (int x = 0; x < 4; ++x) {
            const __half2 h2 = __floats2half2_rn(__uint_as_float(w[x] << 16), __uint_as_float(w[x] & 0xffff0000u));
            hw[x] = *reinterpret_cast<const uint32_t*>(&h2);
          }
          *reinterpret_cast<uint4*>(vop + (size_t)(rbase + row) * D + c * 8) = make_uint4(hw[0], hw[1], hw[2], hw[3]);
        }
      }
      mbar_arrive(&sm.empty[s]);
    }
    // max |v| of the group: warp maxima through shared memory (red[0][0][0..3] is free here)
    for (int o = 16; o > 0; o >>= 1) vabs = fmaxf(vabs, __shfl_xor_sync(0xffffffffu, vabs, o));
    if (lane == 0) sm.red[0][0][warp] = vabs;
    bar_epi();
    if (tid == 0)
      p.vmax[(size_t)bh * nparts + part] = fmaxf(fmaxf(sm.red[0][0][0], sm.red[0][0][1]), fmaxf(sm.red[0][0][2], sm.red[0][0][3]));
    if constexpr (kFirstOrder) {
      if (ok) ok = !epi_any_failed(!wait_bar(&sm.acc_done, 0, &sm.abort, p.status, p.wait_ns));
      if (ok) {
        tc_fence_after();
        const uint32_t trow = tmem + ((uint32_t)(warp * 32) << 16);
        float* out = p.partials + ((size_t)bh * nparts + part) * D * D + (size_t)tid * D;
#pragma unroll
        for (int ch = 0; ch < 4; ++ch) {
          float a[32];
          tmem_ld32(trow + 32 * ch, a);
          tmem_ld_wait();
          if (ntile == 0) {
#pragma unroll
            for (int x = 0; x < 32; ++x) a[x] = 0.f;
          }
#pragma unroll
          for (int x = 0; x < 32; x += 4)
            *reinterpret_cast<float4*>(out + 32 * ch + x) =
                make_float4(a[x] - corr[32 * ch + x], a[x + 1] - corr[32 * ch + x + 1], a[x + 2] - corr[32 * ch + x + 2],
                            a[x + 3] - corr[32 * ch + x + 3]);
        }
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (kFirstOrder && warp == 5) {
    __syncwarp();
    tmem_dealloc(tmem, 128);
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

// ----------------------------------------------------------------------------------------------
// Pass B
// ----------------------------------------------------------------------------------------------
constexpr int kStagesB = 3;
constexpr int kBlocksPerCtaB = 16;

struct alignas(1024) SmemB {
  uint8_t k[kStagesB][kTile];
  uint8_t v[kStagesB][kTile];
  float kbp[kBlocksPerCtaB][128];   // this CTA's centroids kbar_j and value sums vsum_j
  float vsp[kBlocksPerCtaB][128];
  float red[2][4];
  uint64_t full[kStagesB], empty[kStagesB], acc_full[2], acc_empty[2], drain;
  uint32_t tmem_base;
  int abort;
};

// kDiff: also write the per-block first-order operand copy s (H_j - Hbar) (stats with H only); a
// template parameter so that the usual pass keeps its registers for the norms.
template <bool kDiff>
__global__ void __launch_bounds__(kThreads, 1) cov_norm_sm100(const __grid_constant__ KVMaps maps, const PreParams p) {
  extern __shared__ uint8_t smem_raw[];
  SmemB& sm = *reinterpret_cast<SmemB*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int grp = blockIdx.x, bh = blockIdx.y;
  const int jb0 = grp * kBlocksPerCtaB, jb1 = min(p.nb, jb0 + kBlocksPerCtaB);
  const int row0 = jb0 * p.block, row1 = min(p.L, jb1 * p.block);
  const int ntile = (row1 - row0 + 127) / 128;
  const int bpt = 128 / p.block;
  const int ksteps = p.block / 16;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStagesB; ++s) {
      mbar_init(&sm.full[s], 1);
      mbar_init(&sm.empty[s], 129);      // the MMA commit + the 128 threads that copy V out as fp16
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&sm.acc_full[b], 1);
      mbar_init(&sm.acc_empty[b], 128);
    }
    mbar_init(&sm.drain, 1);
    sm.abort = 0;
    fence_mbar_init();
  }
  if (warp == 5) {
    tmem_alloc(&sm.tmem_base, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = sm.tmem_base;

  if (warp == 4) {
    if (lane == 0) {
      int issued = 0;
      bool ok = true;
      for (int t = 0; t < ntile; ++t) {
        const int s = t % kStagesB;
        if (t >= kStagesB &&
            !(ok = wait_bar(&sm.empty[s], ((t / kStagesB) - 1) & 1, &sm.abort, p.status, p.wait_ns)))
          break;
        const int y = row0 + t * 128;
        mbar_expect_tx(&sm.full[s], 2 * kTile);
        tma_load_3d(sm.k[s], &maps.k, &sm.full[s], 0, y, bh);
        tma_load_3d(sm.k[s] + kHalf, &maps.k, &sm.full[s], 64, y, bh);
        tma_load_3d(sm.v[s], &maps.v, &sm.full[s], 0, y, bh);
        tma_load_3d(sm.v[s] + kHalf, &maps.v, &sm.full[s], 64, y, bh);
        ++issued;
      }
      {   // let issued copies land before shared memory is released (normally already landed)
        for (int t = max(0, issued - kStagesB); t < issued; ++t)
          mbar_drain(&sm.full[t % kStagesB], (t / kStagesB) & 1, p.wait_ns);
      }
    }
  } else if (warp == 5) {
    if (lane == 0) {
      bool ok = true;
      for (int t = 0; t < ntile && ok; ++t) {
        const int s = t % kStagesB, buf = t & 1;
        if (!(ok = wait_bar(&sm.full[s], (t / kStagesB) & 1, &sm.abort, p.status, p.wait_ns))) break;
        if (t >= 2 && !(ok = wait_bar(&sm.acc_empty[buf], ((t >> 1) - 1) & 1, &sm.abort, p.status, p.wait_ns))) break;
        tc_fence_after();
        const uint32_t ka = smem_u32(sm.k[s]), va = smem_u32(sm.v[s]);
        for (int b = 0; b < bpt; ++b) {
          const uint32_t d = tmem + (uint32_t)(buf * 256 + b * 128);
          for (int kk = 0; kk < ksteps; ++kk) {
            const uint32_t off = (uint32_t)(b * p.block + kk * 16) * 128;
            mma_ss(d, smem_desc_sw128(ka + off, kHalf, 1024), smem_desc_sw128(va + off, kHalf, 1024), kIdescKV,
                   kk > 0 ? 1u : 0u);
          }
        }
        mma_commit(&sm.empty[s]);
        mma_commit(&sm.acc_full[buf]);
      }
      mma_commit(&sm.drain);      // completes once every MMA above has: TMEM may then be released
      const uint64_t t0 = globaltimer_ns();
      while (!mbar_try_wait(&sm.drain, 0) && globaltimer_ns() - t0 < p.wait_ns) {}
    }
  } else {
    const int a = threadIdx.x;                       // H row a == TMEM lane a
    const uint32_t trow = tmem + ((uint32_t)(warp * 32) << 16);
    const float vinv = 1.f / p.st.vscale[bh];
    __half* vop = reinterpret_cast<__half*>(p.st.v_op) + (size_t)bh * p.L * D;
    __half* vsop = reinterpret_cast<__half*>(p.st.vsum_op);
    {
      // column a of every block's kbar and vsum, all loads issued before the first use; the fp16
      // operand copy vsum / vscale is written here too
      float kv[kBlocksPerCtaB], vv[kBlocksPerCtaB];
#pragma unroll
      for (int jj = 0; jj < kBlocksPerCtaB; ++jj) {
        const size_t so = ((size_t)bh * p.nb + min(jb0 + jj, jb1 - 1)) * D + a;
        kv[jj] = p.st.kbar[so];
        vv[jj] = p.st.vsum[so];
      }
#pragma unroll
      for (int jj = 0; jj < kBlocksPerCtaB; ++jj) {
        sm.kbp[jj][a] = kv[jj];
        sm.vsp[jj][a] = vv[jj];
        if (jb0 + jj < jb1) vsop[((size_t)bh * p.nb + jb0 + jj) * D + a] = __float2half_rn(vv[jj] * vinv);
      }
      bar_epi();
    }
    float hb[D];
    const float* hbar = p.st.hbar + (size_t)bh * D * D + (size_t)a * D;
#pragma unroll
    for (int x = 0; x < D; x += 4) {
      const float4 h4 = *reinterpret_cast<const float4*>(hbar + x);
      hb[x] = h4.x;
      hb[x + 1] = h4.y;
      hb[x + 2] = h4.z;
      hb[x + 3] = h4.w;
    }
    bool ok = true;
    for (int t = 0; t < ntile; ++t) {
      const int buf = t & 1;
      ok = !epi_any_failed(!wait_bar(&sm.acc_full[buf], (t >> 1) & 1, &sm.abort, p.status, p.wait_ns));
      if (!ok) break;
      tc_fence_after();
      {
        // fp16 copy of this tile's values, v / vscale: the H_j MMAs of the tile are done, so the stage
        // has landed and is held until the arrival below; 16-byte chunks, consecutive per thread
        const uint8_t* vt = sm.v[t % kStagesB];
        const int rbase = row0 + t * 128;
        for (int q = a; q < 128 * 16; q += 128) {
          const int row = q >> 4, c = q & 15;
          if (rbase + row >= row1) break;
          const uint4 u = *reinterpret_cast<const uint4*>(vt + (c >> 3) * kHalf + row * 128 + (((c & 7) ^ (row & 7)) << 4));
          const uint32_t w[4] = {u.x, u.y, u.z, u.w};
          uint32_t hw[4];
#pragma unroll
          for (int x = 0; x < 4; ++x) {
            const __half2 h2 = __floats2half2_rn(__uint_as_float(w[x] << 16) * vinv, __uint_as_float(w[x] & 0xffff0000u) * vinv);
            hw[x] = *reinterpret_cast<const uint32_t*>(&h2);
          }
          *reinterpret_cast<uint4*>(vop + (size_t)(rbase + row) * D + c * 8) = make_uint4(hw[0], hw[1], hw[2], hw[3]);
        }
        mbar_arrive(&sm.empty[t % kStagesB]);
      }
      for (int b = 0; b < bpt; ++b) {
        const int j = jb0 + t * bpt + b;
        const bool live = j < jb1;
        const float* vsj = sm.vsp[live ? j - jb0 : 0];
        const float kb = live ? sm.kbp[j - jb0][a] : 0.f;   // 0: a missing block's H stays unused
        const int rb = (t * bpt + b) & 1;                    // red[] alternates between blocks
        float ss = 0.f;
        float* Hout = (live && p.st.H) ? p.st.H + ((size_t)bh * p.nb + j) * D * D + (size_t)a * D : nullptr;
        __nv_bfloat16* Dout = (kDiff && live && p.st.hdiff_op)
                                  ? static_cast<__nv_bfloat16*>(p.st.hdiff_op) + ((size_t)bh * p.nb + j) * D * D + (size_t)a * D
                                  : nullptr;
#pragma unroll
        for (int ch = 0; ch < 4; ++ch) {
          float h[32];
          tmem_ld32(trow + (uint32_t)(buf * 256 + b * 128 + 32 * ch), h);
          tmem_ld_wait();
#pragma unroll
          for (int x = 0; x < 32; ++x) h[x] = fmaf(-kb, vsj[32 * ch + x], h[x]);
          if (Hout) {
#pragma unroll
            for (int x = 0; x < 32; x += 4)
              *reinterpret_cast<float4*>(Hout + 32 * ch + x) = make_float4(h[x], h[x + 1], h[x + 2], h[x + 3]);
          }
#pragma unroll
          for (int x = 0; x < 32; ++x) {
            h[x] -= hb[32 * ch + x];      // H_j - Hbar
            ss = fmaf(h[x], h[x], ss);
          }
          if (kDiff && Dout) {
            // operand copy of the per-block first-order difference: s (H_j - Hbar), row a, bf16
            uint32_t pk[16];
#pragma unroll
            for (int x = 0; x < 32; x += 2) pk[x >> 1] = pack_bf16x2(p.scale * h[x], p.scale * h[x + 1]);
            uint4* dst = reinterpret_cast<uint4*>(Dout + 32 * ch);
#pragma unroll
            for (int x = 0; x < 4; ++x) dst[x] = make_uint4(pk[4 * x], pk[4 * x + 1], pk[4 * x + 2], pk[4 * x + 3]);
          }
        }
        for (int o = 16; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
        if (lane == 0) sm.red[rb][warp] = ss;
        bar_epi();
        if (a == 0 && live) p.st.M[(size_t)bh * p.nb + j] = sqrtf(sm.red[rb][0] + sm.red[rb][1] + sm.red[rb][2] + sm.red[rb][3]);
      }
      tc_fence_before();
      mbar_arrive(&sm.acc_empty[buf]);
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

}  // namespace

cudaError_t launch_precompute_sm100(const Dims& g, const void* q, const void* k, const void* v, const pisa_stats& st,
                                    void* ws, bool first_order, cudaStream_t stream) {
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
  p.wait_ns = kWaitLimitNs;
  const size_t smem_a = sizeof(SmemA) + 1024, smem_b = sizeof(SmemB) + 1024;
  cudaError_t e;
  if ((e = cudaFuncSetAttribute(stats_a_sm100<true>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem_a))) return e;
  if ((e = cudaFuncSetAttribute(stats_a_sm100<false>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem_a))) return e;
  if ((e = cudaFuncSetAttribute(cov_norm_sm100<false>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem_b))) return e;
  if ((e = cudaFuncSetAttribute(cov_norm_sm100<true>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem_b))) return e;
  const int nparts = num_parts(g);
  if (!first_order) {
    stats_a_sm100<false><<<dim3(nparts, g.BH()), kThreads, smem_a, stream>>>(maps, p);
    value_scale_finish<<<dim3(nparts, g.BH()), 256, 0, stream>>>(static_cast<const __nv_bfloat16*>(v), p);
    return cudaGetLastError();
  }
  stats_a_sm100<true><<<dim3(nparts, g.BH()), kThreads, smem_a, stream>>>(maps, p);
  if ((e = launch_hbar_reduce(g, p.partials, nparts, p.vmax, st, stream))) return e;
  const dim3 grid_b((g.nb + kBlocksPerCtaB - 1) / kBlocksPerCtaB, g.BH());
  if (st.hdiff_op)
    cov_norm_sm100<true><<<grid_b, kThreads, smem_b, stream>>>(maps, p);
  else
    cov_norm_sm100<false><<<grid_b, kThreads, smem_b, stream>>>(maps, p);
  return cudaGetLastError();
}

}  // namespace pisa
