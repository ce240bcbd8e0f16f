// Internal: the bodies of the two bf16 pre-computation passes (TMA tiles, tcgen05 contractions),
// shared by their own kernels (precompute_sm100.cu) and by the fused short-sequence kernel
// (short_step_sm100.cu).
#pragma once

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
  int fault = 0;             // test-only fault injection (pisa_testing.h); 0 in normal calls
};

// ----------------------------------------------------------------------------------------------
// Pass A
// ----------------------------------------------------------------------------------------------
// Block sums on the tensor core: for a 128-row tile X (q, k or v) and the 0/1 indicator matrix
// Ind[j][n] = [row n belongs to the j-th block of the tile] (j < 16, K-major in shared memory),
// D[a][j] = sum_n X[n][a] Ind[j][n] is the sum of column a over block j: one M=128, N=16 MMA chain
// per tensor, whose result thread a reads from TMEM lane a.  Products are exact (x * 1) and the
// sums are kept in fp32.
constexpr int kSumCols = 16;                                                    // N of the sum MMAs
constexpr uint32_t kIdescSum = idesc_bf16_f32(128, kSumCols, true, false);      // A = X^T (MN), B = Ind (K)
// TMEM: sum_n k_n v_n^T of a group in one of two 128-column buffers (at 0 and 128, first order only),
// so that one group's epilogue overlaps the next group's MMAs.

// First TMEM column of the two buffers of q, k, v block sums (48 columns each): after the two
// group sums when there are.
__host__ __device__ constexpr uint32_t pass_a_sum_col(bool first_order) { return first_order ? 256u : 0u; }

struct alignas(1024) SmemA {
  uint8_t q[2][kTile];
  uint8_t k[2][kTile];
  uint8_t v[2][kTile];
  uint8_t ind[2][kSumCols * 128];   // indicator, two K halves of [16 rows x 64 bf16], 128B-swizzled
  float cv[2][128];                 // value sums of the last two blocks (rank-1 centring term)
  float red[2][4];                  // per-warp max |v|, alternating between groups
  uint64_t full[2], empty[2], sums_full[2], sums_empty[2], acc_full[2], acc_empty[2], drain;
  uint32_t tmem_base;
  int abort;
};

// TMEM columns pass A allocates (a power of two >= 32): the two group-sum buffers (first order only)
// and the two block-sum buffers.
__host__ __device__ constexpr uint32_t pass_a_tmem_cols(bool first_order) { return first_order ? 512u : 128u; }
static_assert(pass_a_sum_col(true) + 2 * 48 <= pass_a_tmem_cols(true) &&
              pass_a_sum_col(false) + 2 * 48 <= pass_a_tmem_cols(false), "pass A TMEM columns");

// Fills the block indicator for blocks of `block` rows (64: two blocks per 128-row tile, 128: one).
__device__ __forceinline__ void fill_indicator(SmemA& sm, int block) {
  for (int e = threadIdx.x; e < kSumCols * 128; e += blockDim.x) {
    const int j = e >> 7, n = e & 127;
    const int half = n >> 6, nn = n & 63;
    const uint32_t off = (uint32_t)((j >> 3) * 1024 + (j & 7) * 128 + ((((nn >> 3) ^ (j & 7)) << 4)) + (nn & 7) * 2);
    const uint16_t one = 0x3F80u;   // bf16 1.0
    *reinterpret_cast<uint16_t*>(sm.ind[half] + off) = (j == n / block) ? one : (uint16_t)0;
  }
}

__device__ __forceinline__ uint32_t max_u16x2(uint32_t a, uint32_t b) {
  uint32_t r;
  asm("max.u16x2 %0, %1, %2;" : "=r"(r) : "r"(a), "r"(b));
  return r;
}

// max over the 8 bf16 of a 16-byte chunk of |x|, as the bit pattern of a non-negative bf16 in each
// half of the result (clearing the sign makes the bit order the value order)
__device__ __forceinline__ uint32_t absmax8(const uint4& u, uint32_t m) {
  uint32_t r;
  asm("max.u16x2 %0, %1, %2;" : "=r"(r) : "r"(u.x & 0x7fff7fffu), "r"(u.y & 0x7fff7fffu));
  asm("max.u16x2 %0, %1, %2;" : "=r"(r) : "r"(r), "r"(u.z & 0x7fff7fffu));
  asm("max.u16x2 %0, %1, %2;" : "=r"(r) : "r"(r), "r"(u.w & 0x7fff7fffu));
  asm("max.u16x2 %0, %1, %2;" : "=r"(r) : "r"(r), "r"(m));
  return r;
}

// The key blocks, rows and 128-row tiles of pre-computation group u (groups numbered head-major:
// u = bh * ngroups + part, kBlocksPerPart key blocks each).
struct Group {
  int bh, part, jb0, jb1, row0, row1, ntile;
};
__device__ __forceinline__ Group group_of(const PreParams& p, int u, int ngroups) {
  Group g;
  g.bh = u / ngroups;
  g.part = u - g.bh * ngroups;
  g.jb0 = g.part * kBlocksPerPart;
  g.jb1 = min(p.nb, g.jb0 + kBlocksPerPart);
  g.row0 = g.jb0 * p.block;
  g.row1 = min(p.L, g.jb1 * p.block);
  g.ntile = (g.row1 - g.row0 + 127) / 128;
  return g;
}

// kFirstOrder: also accumulate each group's partial sum of H_j (tensor core) for Hbar.  Without it
// (the zeroth-order pre-computation) the CTA writes the fp16 value operand with scale 1 from the V
// tiles it streams, on the chance that the head's value scale is 1; value_scale_finish rewrites it
// when it is not.
//
// Body of pass A for groups [u0, u1) (of `ngroups` per head), one after the other: warps 0-3 take
// the block sums out of TMEM (thread a = column a), write the statistics, keep the rank-1 centring
// term and sweep the V tiles for max |v|; warp 4 loads; warp 5 issues the MMAs into the TMEM
// columns at `tmem` (pass_a_tmem_cols, allocated by the caller); further warps of a larger CTA
// idle.  The tile stream does not stop between groups: the loads and MMAs of the next group run
// while the epilogue writes the previous group's partial sum of H_j (row-major D x D, to
// p.partials + u D^2) out of the other TMEM buffer.  Starts and ends with a CTA-wide barrier; the
// caller owns the TMEM allocation.
template <bool kFirstOrder>
__device__ __forceinline__ void stats_a_body(const KVMaps& maps, const PreParams& p, SmemA& sm, uint32_t tmem,
                                             int u0, int u1, int ngroups) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int bpt = 128 / p.block;

  if (threadIdx.x == 0) {
    for (int s = 0; s < 2; ++s) {
      mbar_init(&sm.full[s], 1);
      mbar_init(&sm.empty[s], 129);        // the MMA commit + the 128 threads that sweep the V tile
      mbar_init(&sm.sums_full[s], 1);
      mbar_init(&sm.sums_empty[s], 128);
      mbar_init(&sm.acc_full[s], 1);
      mbar_init(&sm.acc_empty[s], 128);
    }
    mbar_init(&sm.drain, 1);
    sm.abort = 0;
    fence_mbar_init();
  }
  fill_indicator(sm, p.block);
  fence_async_shared();                   // the indicator is read by the tensor core (async proxy)
  tc_fence_before();
  __syncthreads();
  tc_fence_after();

  // Tiles are counted over all groups of the CTA (g): stage and block-sum buffer g & 1.  Group i of
  // the CTA accumulates into group-sum buffer i & 1.
  if (warp == 4) {
    if (lane == 0) {
      int g = 0;
      bool ok = true;
      // fault 2 (tests only): the first tile is never loaded, so the MMA warp's wait for it runs out
      const int skipped = p.fault == 2 ? 0 : -1;
      for (int u = u0; u < u1 && ok; ++u) {
        const Group gr = group_of(p, u, ngroups);
        for (int t = 0; t < gr.ntile; ++t, ++g) {
          const int s = g & 1;
          if (g >= 2 && !(ok = wait_bar(&sm.empty[s], ((g >> 1) - 1) & 1, &sm.abort, p.status, p.wait_ns))) break;
          if (g == skipped) continue;
          const int y = gr.row0 + t * 128;
          mbar_expect_tx(&sm.full[s], 3 * kTile);
          tma_load_3d(sm.q[s], &maps.q, &sm.full[s], 0, y, gr.bh);
          tma_load_3d(sm.q[s] + kHalf, &maps.q, &sm.full[s], 64, y, gr.bh);
          tma_load_3d(sm.k[s], &maps.k, &sm.full[s], 0, y, gr.bh);
          tma_load_3d(sm.k[s] + kHalf, &maps.k, &sm.full[s], 64, y, gr.bh);
          tma_load_3d(sm.v[s], &maps.v, &sm.full[s], 0, y, gr.bh);
          tma_load_3d(sm.v[s] + kHalf, &maps.v, &sm.full[s], 64, y, gr.bh);
        }
      }
      {   // let issued copies land before shared memory is released (normally already landed)
        for (int i = max(0, g - 2); i < g; ++i)
          if (i != skipped) mbar_drain(&sm.full[i & 1], (i >> 1) & 1, p.wait_ns);
      }
    }
  } else if (warp == 5) {
    if (lane == 0) {
      bool ok = true;
      const uint32_t ia = smem_u32(sm.ind[0]);
      int g = 0;
      for (int u = u0, i = 0; u < u1 && ok; ++u, ++i) {
        const Group gr = group_of(p, u, ngroups);
        const uint32_t acc = tmem + (uint32_t)(i & 1) * 128;
        if (kFirstOrder && i >= 2 &&
            !(ok = wait_bar(&sm.acc_empty[i & 1], ((i >> 1) - 1) & 1, &sm.abort, p.status, p.wait_ns)))
          break;
        for (int t = 0; t < gr.ntile; ++t, ++g) {
          const int s = g & 1;
          if (!(ok = wait_bar(&sm.full[s], (g >> 1) & 1, &sm.abort, p.status, p.wait_ns))) break;
          if (g >= 2 && !(ok = wait_bar(&sm.sums_empty[s], ((g >> 1) - 1) & 1, &sm.abort, p.status, p.wait_ns))) break;
          tc_fence_after();
          const uint32_t qa = smem_u32(sm.q[s]), ka = smem_u32(sm.k[s]), va = smem_u32(sm.v[s]);
          if (kFirstOrder) {
#pragma unroll
            for (int kk = 0; kk < 8; ++kk)
              mma_ss(acc, smem_desc_sw128(ka + kk * 2048, kHalf, 1024), smem_desc_sw128(va + kk * 2048, kHalf, 1024),
                     kIdescKV, (t > 0 || kk > 0) ? 1u : 0u);
          }
          // block sums of q, k, v: 16 rows (one K step) of the tile and the matching 16 columns of
          // the indicator per instruction
          const uint32_t dsum = tmem + pass_a_sum_col(kFirstOrder) + (uint32_t)s * 48;
#pragma unroll
          for (int x = 0; x < 3; ++x) {
            const uint32_t xa = x == 0 ? qa : (x == 1 ? ka : va);
#pragma unroll
            for (int kk = 0; kk < 8; ++kk)
              mma_ss(dsum + 16 * x, smem_desc_sw128(xa + kk * 2048, kHalf, 1024),
                     smem_desc_sw128(ia + (kk >> 2) * (kSumCols * 128) + (kk & 3) * 32, 16, 1024), kIdescSum,
                     kk > 0 ? 1u : 0u);
          }
          mma_commit(&sm.sums_full[s]);
          mma_commit(&sm.empty[s]);
        }
        if (kFirstOrder && ok) mma_commit(&sm.acc_full[i & 1]);
      }
      mma_commit(&sm.drain);      // completes once every MMA above has: TMEM may then be released
      mbar_drain(&sm.drain, 0, p.wait_ns);
    }
  } else if (warp < 4) {
    const int tid = threadIdx.x;            // column a of q, k, v == TMEM lane a
    const uint32_t trow = tmem + ((uint32_t)(warp * 32) << 16);
    bool ok = true;
    int g = 0, nblk = 0;
    for (int u = u0, i = 0; u < u1 && ok; ++u, ++i) {
      const Group gr = group_of(p, u, ngroups);
      uint64_t corr2[kFirstOrder ? D / 2 : 1];    // the group's centring term, packed pairs of columns
#pragma unroll
      for (int c = 0; c < (kFirstOrder ? D / 2 : 1); ++c) corr2[c] = f2_pack(0.f, 0.f);
      uint32_t vabs = 0u;                         // two packed non-negative bf16
      __half* vop = reinterpret_cast<__half*>(p.st.v_op) + (size_t)gr.bh * p.L * D;
      for (int t = 0; t < gr.ntile; ++t, ++g) {
        const int s = g & 1;
        ok = !epi_any_failed(!wait_bar(&sm.full[s], (g >> 1) & 1, &sm.abort, p.status, p.wait_ns));
        if (!ok) break;
        // max |v| over the tile (and, zeroth order only, the fp16 value operand with scale 1):
        // 16-byte chunks of the swizzled V tile, consecutive chunks per thread.  A tile reaches past
        // its group only at the end of the head, where the tile load fills zeros, so the maximum
        // needs no row bound (only the head's maximum is used): the first-order sweep is unrolled
        // into four independent running maxima.
        if constexpr (kFirstOrder) {
          uint32_t m4[4] = {vabs, 0u, 0u, 0u};
#pragma unroll
          for (int x = 0; x < 16; ++x) {
            const int qq = tid + 128 * x, row = qq >> 4, c = qq & 15;
            const uint4 uu = *reinterpret_cast<const uint4*>(sm.v[s] + (c >> 3) * kHalf + row * 128 + (((c & 7) ^ (row & 7)) << 4));
            m4[x & 3] = absmax8(uu, m4[x & 3]);
          }
          vabs = max_u16x2(max_u16x2(m4[0], m4[1]), max_u16x2(m4[2], m4[3]));
        } else {
          const int rbase = gr.row0 + t * 128;
          for (int qq = tid; qq < 128 * 16; qq += 128) {
            const int row = qq >> 4, c = qq & 15;
            if (rbase + row >= gr.row1) break;
            const uint4 uu = *reinterpret_cast<const uint4*>(sm.v[s] + (c >> 3) * kHalf + row * 128 + (((c & 7) ^ (row & 7)) << 4));
            vabs = absmax8(uu, vabs);
            const uint32_t w[4] = {uu.x, uu.y, uu.z, uu.w};
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
        ok = !epi_any_failed(!wait_bar(&sm.sums_full[s], (g >> 1) & 1, &sm.abort, p.status, p.wait_ns));
        if (!ok) break;
        tc_fence_after();
        uint32_t sq[2], sk[2], sv[2];
        const uint32_t dsum = trow + pass_a_sum_col(kFirstOrder) + (uint32_t)s * 48;
        tmem_ld2(dsum, sq);
        tmem_ld2(dsum + 16, sk);
        tmem_ld2(dsum + 32, sv);
        tmem_ld_wait();
        tc_fence_before();
        mbar_arrive(&sm.sums_empty[s]);
        for (int b = 0; b < bpt; ++b) {
          const int j = gr.jb0 + t * bpt + b;
          if (j >= gr.jb1) break;
          const float inv = 1.f / (float)block_count(j, p.L, p.block);
          // (bpt <= 2: select rather than index, so the sums stay in registers)
          const float qs = __uint_as_float(b ? sq[1] : sq[0]), ks = __uint_as_float(b ? sk[1] : sk[0]),
                      vs = __uint_as_float(b ? sv[1] : sv[0]);
          const size_t so = ((size_t)gr.bh * p.nb + j) * D + tid;
          p.st.qbar[so] = qs * inv;
          p.st.kbar[so] = ks * inv;
          p.st.vsum[so] = vs;
          reinterpret_cast<__nv_bfloat16*>(p.st.kbar_op)[so] = __float2bfloat16_rn(ks * inv);
          if constexpr (kFirstOrder) {
            // rank-1 centring term sum_j kbar_j vsum_j^T: row tid needs every column of vsum_j
            const int pb = nblk & 1;
            sm.cv[pb][tid] = vs;
            bar_epi();
            const uint64_t ka2 = f2_pack(ks * inv, ks * inv);
#pragma unroll
            for (int x = 0; x < D; x += 4) {
              const float4 c4 = *reinterpret_cast<const float4*>(&sm.cv[pb][x]);
              corr2[x / 2] = f2_fma(ka2, f2_pack(c4.x, c4.y), corr2[x / 2]);
              corr2[x / 2 + 1] = f2_fma(ka2, f2_pack(c4.z, c4.w), corr2[x / 2 + 1]);
            }
          }
          ++nblk;
        }
      }
      if (!ok) break;
      // max |v| of the group: warp maxima through shared memory (two buffers: a warp that runs
      // ahead into the next group cannot overwrite what thread 0 has not read yet)
      {
        float va = fmaxf(__uint_as_float(vabs << 16), __uint_as_float(vabs & 0xffff0000u));
        for (int o = 16; o > 0; o >>= 1) va = fmaxf(va, __shfl_xor_sync(0xffffffffu, va, o));
        if (lane == 0) sm.red[i & 1][warp] = va;
        bar_epi();
        if (tid == 0)
          p.vmax[u] = fmaxf(fmaxf(sm.red[i & 1][0], sm.red[i & 1][1]), fmaxf(sm.red[i & 1][2], sm.red[i & 1][3]));
      }
      if constexpr (kFirstOrder) {
        ok = !epi_any_failed(!wait_bar(&sm.acc_full[i & 1], (i >> 1) & 1, &sm.abort, p.status, p.wait_ns));
        if (!ok) break;
        tc_fence_after();
        float* out = p.partials + (size_t)u * D * D + (size_t)tid * D;
#pragma unroll
        for (int ch = 0; ch < 4; ++ch) {
          float a[32];
          tmem_ld32(trow + (uint32_t)(i & 1) * 128 + 32 * ch, a);
          tmem_ld_wait();
#pragma unroll
          for (int x = 0; x < 32; x += 4) {
            float c0, c1, c2, c3;
            f2_unpack(corr2[(32 * ch + x) / 2], c0, c1);
            f2_unpack(corr2[(32 * ch + x) / 2 + 1], c2, c3);
            *reinterpret_cast<float4*>(out + 32 * ch + x) = make_float4(a[x] - c0, a[x + 1] - c1, a[x + 2] - c2, a[x + 3] - c3);
          }
        }
        tc_fence_before();
        mbar_arrive(&sm.acc_empty[i & 1]);
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
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
//
// Body of pass B for groups [u0, u1) (of `ngroups` per head, kBlocksPerCtaB key blocks each), one
// after the other: warps 0-3 epilogue, warp 4 loads, warp 5 issues the MMAs into the 512 TMEM
// columns at `tmem` (allocated by the caller); further warps of a larger CTA idle.  The tile
// stream does not stop between groups (the epilogue's set-up of a group, its centroids and value
// sums, overlaps the loads and MMAs of the group's first tiles); the Hbar row each epilogue thread
// keeps in registers is reloaded only when the head changes.  Starts and ends with a CTA-wide
// barrier.
template <bool kDiff>
__device__ __forceinline__ void cov_norm_body(const KVMaps& maps, const PreParams& p, SmemB& sm, uint32_t tmem,
                                              int u0, int u1, int ngroups) {
  static_assert(kBlocksPerCtaB == kBlocksPerPart, "pass B groups are pass A groups");
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
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
  tc_fence_before();
  __syncthreads();
  tc_fence_after();

  // Tiles are counted over all groups of the CTA (g): stage g % kStagesB, TMEM buffer g & 1.
  if (warp == 4) {
    if (lane == 0) {
      int g = 0;
      bool ok = true;
      for (int u = u0; u < u1 && ok; ++u) {
        const Group gr = group_of(p, u, ngroups);
        for (int t = 0; t < gr.ntile; ++t, ++g) {
          const int s = g % kStagesB;
          if (g >= kStagesB &&
              !(ok = wait_bar(&sm.empty[s], ((g / kStagesB) - 1) & 1, &sm.abort, p.status, p.wait_ns)))
            break;
          const int y = gr.row0 + t * 128;
          mbar_expect_tx(&sm.full[s], 2 * kTile);
          tma_load_3d(sm.k[s], &maps.k, &sm.full[s], 0, y, gr.bh);
          tma_load_3d(sm.k[s] + kHalf, &maps.k, &sm.full[s], 64, y, gr.bh);
          tma_load_3d(sm.v[s], &maps.v, &sm.full[s], 0, y, gr.bh);
          tma_load_3d(sm.v[s] + kHalf, &maps.v, &sm.full[s], 64, y, gr.bh);
        }
      }
      {   // let issued copies land before shared memory is released (normally already landed)
        for (int i = max(0, g - kStagesB); i < g; ++i) mbar_drain(&sm.full[i % kStagesB], (i / kStagesB) & 1, p.wait_ns);
      }
    }
  } else if (warp == 5) {
    if (lane == 0) {
      bool ok = true;
      int g = 0;
      for (int u = u0; u < u1 && ok; ++u) {
        const Group gr = group_of(p, u, ngroups);
        for (int t = 0; t < gr.ntile; ++t, ++g) {
          const int s = g % kStagesB, buf = g & 1;
          if (!(ok = wait_bar(&sm.full[s], (g / kStagesB) & 1, &sm.abort, p.status, p.wait_ns))) break;
          if (g >= 2 && !(ok = wait_bar(&sm.acc_empty[buf], ((g >> 1) - 1) & 1, &sm.abort, p.status, p.wait_ns))) break;
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
      }
      mma_commit(&sm.drain);      // completes once every MMA above has: TMEM may then be released
      const uint64_t t0 = globaltimer_ns();
      while (!mbar_try_wait(&sm.drain, 0) && globaltimer_ns() - t0 < p.wait_ns) {}
    }
  } else if (warp < 4) {
    // The loads and MMAs above read only K and V; everything below reads what the kernels before
    // this one wrote (the centroids, value sums, Hbar and value scale).  When this kernel was
    // launched as a programmatic dependent of those, it may have started before they finished.
    griddep_wait();
    const int a = threadIdx.x;                       // H row a == TMEM lane a
    const uint32_t trow = tmem + ((uint32_t)(warp * 32) << 16);
    __half* vsop = reinterpret_cast<__half*>(p.st.vsum_op);
    uint64_t nhb[D / 2];                             // row a of -Hbar of the current head, packed pairs
    float vinv = 1.f;
    int cur_bh = -1;
    bool ok = true;
    int g = 0, nblk = 0;
    for (int u = u0; u < u1 && ok; ++u) {
      const Group gr = group_of(p, u, ngroups);
      const int bh = gr.bh;
      {
        // column a of every block's kbar and vsum, all loads issued before the first use; the fp16
        // operand copy vsum / vscale is written here too.  (Every thread is past the previous
        // group's last reads of kbp / vsp: each block ends at a barrier of the 128 threads.)
        if (bh != cur_bh) vinv = 1.f / p.st.vscale[bh];
        float kv[kBlocksPerCtaB], vv[kBlocksPerCtaB];
#pragma unroll
        for (int jj = 0; jj < kBlocksPerCtaB; ++jj) {
          const size_t so = ((size_t)bh * p.nb + min(gr.jb0 + jj, gr.jb1 - 1)) * D + a;
          kv[jj] = p.st.kbar[so];
          vv[jj] = p.st.vsum[so];
        }
#pragma unroll
        for (int jj = 0; jj < kBlocksPerCtaB; ++jj) {
          sm.kbp[jj][a] = kv[jj];
          sm.vsp[jj][a] = vv[jj];
          if (gr.jb0 + jj < gr.jb1) vsop[((size_t)bh * p.nb + gr.jb0 + jj) * D + a] = __float2half_rn(vv[jj] * vinv);
        }
        bar_epi();
      }
      if (bh != cur_bh) {
        // row a of -Hbar as packed pairs (f32x2 arithmetic below: one instruction per two columns)
        const float* hbar = p.st.hbar + (size_t)bh * D * D + (size_t)a * D;
#pragma unroll
        for (int x = 0; x < D; x += 4) {
          const float4 h4 = *reinterpret_cast<const float4*>(hbar + x);
          nhb[x / 2] = f2_pack(-h4.x, -h4.y);
          nhb[x / 2 + 1] = f2_pack(-h4.z, -h4.w);
        }
        cur_bh = bh;
      }
      __half* vop = reinterpret_cast<__half*>(p.st.v_op) + (size_t)bh * p.L * D;
      for (int t = 0; t < gr.ntile; ++t, ++g) {
        const int buf = g & 1;
        ok = !epi_any_failed(!wait_bar(&sm.acc_full[buf], (g >> 1) & 1, &sm.abort, p.status, p.wait_ns));
        if (!ok) break;
        tc_fence_after();
        {
          // fp16 copy of this tile's values, v / vscale: the H_j MMAs of the tile are done, so the
          // stage has landed and is held until the arrival below; 16-byte chunks, consecutive per
          // thread, unrolled (the row bound only bites in the last tile of a head)
          const uint8_t* vt = sm.v[g % kStagesB];
          const int rbase = gr.row0 + t * 128;
#pragma unroll 4
          for (int it = 0; it < 16; ++it) {
            const int q = a + 128 * it, row = q >> 4, c = q & 15;
            const uint4 uu = *reinterpret_cast<const uint4*>(vt + (c >> 3) * kHalf + row * 128 + (((c & 7) ^ (row & 7)) << 4));
            const uint32_t w[4] = {uu.x, uu.y, uu.z, uu.w};
            uint32_t hw[4];
#pragma unroll
            for (int x = 0; x < 4; ++x) {
              float lo = __uint_as_float(w[x] << 16), hi = __uint_as_float(w[x] & 0xffff0000u);
              if (vinv != 1.f) {         // (a power of two: the scaling is exact)
                lo *= vinv;
                hi *= vinv;
              }
              hw[x] = pack_f16x2(lo, hi);
            }
            if (rbase + row < gr.row1)
              *reinterpret_cast<uint4*>(vop + (size_t)(rbase + row) * D + c * 8) = make_uint4(hw[0], hw[1], hw[2], hw[3]);
          }
          mbar_arrive(&sm.empty[g % kStagesB]);
        }
        for (int b = 0; b < bpt; ++b) {
          const int j = gr.jb0 + t * bpt + b;
          const bool live = j < gr.jb1;
          const float* vsj = sm.vsp[live ? j - gr.jb0 : 0];
          const float kb = live ? sm.kbp[j - gr.jb0][a] : 0.f;   // 0: a missing block's H stays unused
          const int rb = nblk & 1;                                // red[] alternates between blocks
          ++nblk;
          const uint64_t nkb2 = f2_pack(-kb, -kb);
          uint64_t ss2 = f2_pack(0.f, 0.f);
          float* Hout = (live && p.st.H) ? p.st.H + ((size_t)bh * p.nb + j) * D * D + (size_t)a * D : nullptr;
          __nv_bfloat16* Dout = (kDiff && live && p.st.hdiff_op)
                                    ? static_cast<__nv_bfloat16*>(p.st.hdiff_op) + ((size_t)bh * p.nb + j) * D * D + (size_t)a * D
                                    : nullptr;
#pragma unroll
          for (int ch = 0; ch < 4; ++ch) {
            float h[32];
            tmem_ld32(trow + (uint32_t)(buf * 256 + b * 128 + 32 * ch), h);
            tmem_ld_wait();
            // H_j = D - kbar_j vsum_j^T, then H_j - Hbar and its squares, two columns per instruction
            uint64_t h2[16];
#pragma unroll
            for (int x = 0; x < 32; x += 4) {
              const float4 v4 = *reinterpret_cast<const float4*>(vsj + 32 * ch + x);
              h2[x / 2] = f2_fma(nkb2, f2_pack(v4.x, v4.y), f2_pack(h[x], h[x + 1]));
              h2[x / 2 + 1] = f2_fma(nkb2, f2_pack(v4.z, v4.w), f2_pack(h[x + 2], h[x + 3]));
            }
            if (Hout) {
#pragma unroll
              for (int x = 0; x < 32; x += 4) {
                float a0, a1, a2, a3;
                f2_unpack(h2[x / 2], a0, a1);
                f2_unpack(h2[x / 2 + 1], a2, a3);
                *reinterpret_cast<float4*>(Hout + 32 * ch + x) = make_float4(a0, a1, a2, a3);
              }
            }
#pragma unroll
            for (int x = 0; x < 16; ++x) {
              h2[x] = f2_add(h2[x], nhb[16 * ch + x]);      // H_j - Hbar
              ss2 = f2_fma(h2[x], h2[x], ss2);
            }
#pragma unroll
            for (int x = 0; x < 32; x += 2) f2_unpack(h2[x / 2], h[x], h[x + 1]);
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
          float ss0, ss1;
          f2_unpack(ss2, ss0, ss1);
          float ss = ss0 + ss1;
          for (int o = 16; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
          if (lane == 0) sm.red[rb][warp] = ss;
          bar_epi();
          if (a == 0 && live) p.st.M[(size_t)bh * p.nb + j] = sqrtf(sm.red[rb][0] + sm.red[rb][1] + sm.red[rb][2] + sm.red[rb][3]);
        }
        tc_fence_before();
        mbar_arrive(&sm.acc_empty[buf]);
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
}

}  // namespace
}  // namespace pisa
