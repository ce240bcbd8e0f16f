// Per-block first-order correction for sm_100a: TMA + tcgen05 (TMEM accumulators).
//
// "PISA: Piecewise Sparse Attention Is Wiser for Efficient Diffusion Transformers", §2 핵심 알고리즘:
// the first-order term of an unselected block j is s (q_t H_j) alpha_tj; the method replaces every
// H_j by their mean Hbar so that no block's d x d matrix has to be loaded.  This kernel measures
// what that costs: after the attention kernel (global Hbar) has left its output o_t in fp32 and each
// row's softmax offset and 1/D_t in the workspace, it writes
//     o_t = bf16( o_t + s sum_{j in U_i} alpha_tj q_t (H_j - Hbar) / D_t ),   alpha_tj = exp(s q_t.kbar_j - offset_t)
// the per-block first-order result, rounded to bf16 once.
//
// Mapping onto B200 (one CTA = one 128-row query tile, the same tiles and query-block pairs as the
// attention kernel; one CTA per SM, 512 TMEM columns):
//   * C = Q kbar^T for 128 centroids at a time (one tcgen05 MMA chain, N = 128) into TMEM.
//   * For each block j that the tile's query blocks did not both select, the four row warps build
//     W_j = alpha_tj q_t (one row per thread, bf16, q_t held in registers) in TMEM, and the MMA warp
//     accumulates O += W_j (s (H_j - Hbar)), A = W_j from TMEM, B = the block's 128 x 128 bf16
//     matrix streamed by TMA.  W slots (TMEM) and matrix stages (shared memory) form one ring of
//     four, so building the next W and loading the next matrices overlap the current MMAs.  Rows whose own query block selected j get alpha = 0.
//   * The epilogue reads O from TMEM, adds the row's fp32 attention output and writes bf16.
// Warp roles: warps 0-3 W builders + epilogue (TMEM lanes 0-127), warp 4 TMA producer, warp 5 MMA
// issuer and TMEM owner.  Every mbarrier wait is bounded; on a timeout the CTA sets the status
// word, drains its own copies and MMAs, frees TMEM and leaves its rows of o unwritten.
#include <cuda.h>

#include "common.cuh"
#include "sm100.cuh"

namespace pisa {
namespace {
using namespace sm100;

constexpr int D = 128;
constexpr int kThreads = 192;
constexpr int kHalf = 128 * 64 * 2;        // 128 rows x 64 bf16 columns, 128B-swizzled: 16 KB
constexpr int kTileBytes = 2 * kHalf;
// One ring of kR slots, each a W buffer in TMEM and a per-block matrix in shared memory, with one
// "full" barrier (the producer's TMA bytes plus the 128 W builders' arrivals) and one "empty"
// barrier (the MMAs' commit): the MMA warp waits once per block.
constexpr int kR = 4;
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kColC = 0, kColW = 128, kColO = 128 + 64 * kR;   // C: 128 cols, W: kR x 64, O: 128
static_assert(kColO + 128 <= kTmemCols, "TMEM columns");
constexpr int kWords = 128;                // selection bitmap words (nb <= 4096)
constexpr int kAlphaStride = 33;

struct alignas(1024) Smem {
  uint8_t q[kTileBytes];
  uint8_t kb[kTileBytes];
  uint8_t h[kR][kTileBytes];
  float alpha[128 * kAlphaStride];          // alpha of the current 32 centroids, one row per thread
  uint64_t bar_q, bar_kfull, bar_kempty, bar_cfull, bar_cempty;
  uint64_t bar_full[kR], bar_empty[kR];
  uint64_t bar_final, bar_drain;
  uint32_t tmem_base;
  int abort;
  int nproc;
  uint32_t bitsA[kWords];
  uint32_t bitsB[kWords];
};

struct Params {
  int L, nb, block, keep_k;
  float scale_log2;
  const int32_t* sel;
  const int32_t* order;
  const float2* rowstats;
  const float* o32;          // [B*H][L][D] attention output with the global first-order term, fp32
  __nv_bfloat16* o;
  int* status;
  unsigned long long wait_ns;
};

__device__ __forceinline__ uint32_t mul_bf16x2(uint32_t a, uint32_t b) {
  uint32_t d;
  asm("mul.rn.bf16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
  return d;
}

// Blocks of the 32 starting at 32*w that the tile processes: inside [0, nb) and not selected by
// both of its query blocks.
__device__ __forceinline__ uint32_t proc_word(const Smem& sm, int w, int nb) {
  const int r = nb - 32 * w;
  const uint32_t valid = r >= 32 ? 0xffffffffu : (r > 0 ? ((1u << r) - 1u) : 0u);
  return valid & ~(sm.bitsA[w] & sm.bitsB[w]);
}

// o row = bf16(o32 row + add[0..127]) for the 32 columns starting at 32*ch
__device__ __forceinline__ void store_row32(const Params& p, size_t row, int ch, const float* add) {
  const float4* src = reinterpret_cast<const float4*>(p.o32 + row * D + 32 * ch);
  uint4* dst = reinterpret_cast<uint4*>(p.o + row * D + 32 * ch);
#pragma unroll
  for (int x = 0; x < 4; ++x) {
    const float4 a = src[2 * x], b = src[2 * x + 1];
    dst[x] = make_uint4(pack_bf16x2(a.x + add[8 * x], a.y + add[8 * x + 1]),
                        pack_bf16x2(a.z + add[8 * x + 2], a.w + add[8 * x + 3]),
                        pack_bf16x2(b.x + add[8 * x + 4], b.y + add[8 * x + 5]),
                        pack_bf16x2(b.z + add[8 * x + 6], b.w + add[8 * x + 7]));
  }
}

__device__ __forceinline__ bool wait_or_abort(Smem& sm, uint64_t* bar, uint32_t parity, const Params& p) {
  if (mbar_wait_bounded(bar, parity, &sm.abort, p.wait_ns)) return true;
  *reinterpret_cast<volatile int*>(&sm.abort) = 1;
  set_status(p.status, PISA_DEVERR_WAIT_TIMEOUT);
  return false;
}

// Selection bitmap of query block qi (out-of-range entries are skipped; the attention kernel of
// the same call has reported them).
__device__ void build_bits(uint32_t* bits, const Params& p, int bh, int qi) {
  const int32_t* row = p.sel + ((size_t)bh * p.nb + qi) * p.keep_k;
  for (int e = threadIdx.x; e < p.keep_k; e += kThreads) {
    const int j = row[e];
    if (j >= 0 && j < p.nb) atomicOr(&bits[j >> 5], 1u << (j & 31));
  }
}

__global__ void __launch_bounds__(kThreads, 1)
perblock_sm100(const __grid_constant__ AttnMaps maps, const __grid_constant__ CUtensorMap hmap, const Params p) {
  extern __shared__ uint8_t smem_raw[];
  Smem& sm = *reinterpret_cast<Smem*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int tile = blockIdx.x, bh = blockIdx.y;
  const bool pair = p.block == 64;

  int qa, qb;
  bool has_b = false;
  if (pair) {
    const int ia = 2 * tile, ib = 2 * tile + 1;
    qa = p.order ? p.order[(size_t)bh * p.nb + ia] : ia;
    has_b = ib < p.nb;
    qb = has_b ? (p.order ? p.order[(size_t)bh * p.nb + ib] : ib) : qa;
  } else {
    qa = qb = tile;
  }
  if (qa < 0 || qa >= p.nb || qb < 0 || qb >= p.nb) return;    // reported by the attention kernel

  for (int w = threadIdx.x; w < kWords; w += kThreads) { sm.bitsA[w] = 0u; sm.bitsB[w] = 0u; }
  __syncthreads();
  build_bits(sm.bitsA, p, bh, qa);
  if (has_b) build_bits(sm.bitsB, p, bh, qb);
  __syncthreads();
  if (!has_b)
    for (int w = threadIdx.x; w < kWords; w += kThreads) sm.bitsB[w] = sm.bitsA[w];
  __syncthreads();
  if (warp == 0) {
    int cnt = 0;
    for (int w = lane; w < kWords; w += 32) cnt += __popc(proc_word(sm, w, p.nb));
    for (int o = 16; o > 0; o >>= 1) cnt += __shfl_xor_sync(0xffffffffu, cnt, o);
    if (lane == 0) sm.nproc = cnt;
  }
  if (threadIdx.x == 0) {
    mbar_init(&sm.bar_q, 1);
    mbar_init(&sm.bar_kfull, 1);
    mbar_init(&sm.bar_kempty, 1);
    mbar_init(&sm.bar_cfull, 1);
    mbar_init(&sm.bar_cempty, 128);
    for (int i = 0; i < kR; ++i) {
      mbar_init(&sm.bar_full[i], 129);     // the producer's arrive.expect_tx + 128 W builders
      mbar_init(&sm.bar_empty[i], 1);      // the MMAs' commit
    }
    mbar_init(&sm.bar_final, 1);
    mbar_init(&sm.bar_drain, 1);
    sm.abort = 0;
    fence_mbar_init();
  }
  __syncthreads();
  if (sm.nproc == 0) {
    // every block of this tile was attended exactly: nothing to add, only the rounding to bf16
    if (threadIdx.x < 128) {
      const int r = threadIdx.x;
      const bool upper = pair && r >= 64;
      const int myq = upper ? qb : qa, rloc = pair ? (r & 63) : r;
      if (rloc < block_count(myq, p.L, p.block) && (!upper || has_b)) {
        const float zero[32] = {};
        for (int ch = 0; ch < 4; ++ch) store_row32(p, (size_t)bh * p.L + (size_t)myq * p.block + rloc, ch, zero);
      }
    }
    return;
  }
  if (warp == 5) {
    tmem_alloc(&sm.tmem_base, kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = sm.tmem_base;
  const int nct = (p.nb + 127) / 128;

  if (warp == 4) {
    // =============================== TMA producer ===============================
    if (lane == 0) {
      tma_prefetch_desc(&maps.q);
      tma_prefetch_desc(&maps.kbar);
      tma_prefetch_desc(&hmap);
      mbar_expect_tx(&sm.bar_q, kTileBytes);
      tma_load_3d(sm.q, &maps.q, &sm.bar_q, 0, qa * p.block, bh);
      tma_load_3d(sm.q + kHalf, &maps.q, &sm.bar_q, 64, qa * p.block, bh);
      if (pair) {
        tma_load_3d(sm.q + 64 * 128, &maps.q, &sm.bar_q, 0, qb * p.block, bh);
        tma_load_3d(sm.q + kHalf + 64 * 128, &maps.q, &sm.bar_q, 64, qb * p.block, bh);
      }
      int issued_k = 0, issued_h = 0;
      bool ok = true;
      for (int ct = 0; ct < nct && ok; ++ct) {
        if (ct > 0 && !(ok = wait_or_abort(sm, &sm.bar_kempty, (ct - 1) & 1, p))) break;
        mbar_expect_tx(&sm.bar_kfull, kTileBytes);
        tma_load_3d(sm.kb, &maps.kbar, &sm.bar_kfull, 0, ct * 128, bh);
        tma_load_3d(sm.kb + kHalf, &maps.kbar, &sm.bar_kfull, 64, ct * 128, bh);
        ++issued_k;
        for (int w = 4 * ct; w < 4 * ct + 4 && ok; ++w) {
          for (uint32_t pm = proc_word(sm, w, p.nb); pm; pm &= pm - 1) {
            const int j = 32 * w + __ffs(pm) - 1;
            const int s = issued_h % kR;
            if (issued_h >= kR && !(ok = wait_or_abort(sm, &sm.bar_empty[s], ((issued_h / kR) - 1) & 1, p)))
              break;
            mbar_expect_tx(&sm.bar_full[s], kTileBytes);
            tma_load_3d(sm.h[s], &hmap, &sm.bar_full[s], 0, j * D, bh);
            tma_load_3d(sm.h[s] + kHalf, &hmap, &sm.bar_full[s], 64, j * D, bh);
            ++issued_h;
          }
        }
      }
      {
        // every copy issued must land before this CTA's shared memory is released (normally the
        // MMA warp has already waited for all of them)
        // (each wait with its own deadline)
        mbar_drain(&sm.bar_q, 0, p.wait_ns);
        if (issued_k > 0) mbar_drain(&sm.bar_kfull, (issued_k - 1) & 1, p.wait_ns);
        for (int i = max(0, issued_h - kR); i < issued_h; ++i) mbar_drain(&sm.bar_full[i % kR], (i / kR) & 1, p.wait_ns);
      }
    }
  } else if (warp == 5) {
    // =============================== MMA issuer ===============================
    if (lane == 0) {
      const uint32_t idesc_c = idesc_bf16_f32(128, 128, false, false);
      const uint32_t idesc_h = idesc_bf16_f32(128, 128, false, true);
      const uint64_t qd = smem_desc_sw128(smem_u32(sm.q), 16, 1024);
      const uint64_t kd = smem_desc_sw128(smem_u32(sm.kb), 16, 1024);
      bool ok = wait_or_abort(sm, &sm.bar_q, 0, p);
      int n = 0;
      for (int ct = 0; ct < nct && ok; ++ct) {
        if (!(ok = wait_or_abort(sm, &sm.bar_kfull, ct & 1, p))) break;
        if (ct > 0 && !(ok = wait_or_abort(sm, &sm.bar_cempty, (ct - 1) & 1, p))) break;
        tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
          const uint32_t off = ((kk >> 2) * kHalf + (kk & 3) * 32) >> 4;
          mma_ss(tmem + kColC, qd + off, kd + off, idesc_c, kk > 0 ? 1u : 0u);
        }
        mma_commit(&sm.bar_kempty);
        mma_commit(&sm.bar_cfull);
        for (int w = 4 * ct; w < 4 * ct + 4 && ok; ++w) {
          for (uint32_t pm = proc_word(sm, w, p.nb); pm; pm &= pm - 1) {
            const int slot = n % kR, s = slot;
            if (!(ok = wait_or_abort(sm, &sm.bar_full[slot], (n / kR) & 1, p))) break;
            tc_fence_after();
            const uint64_t hd = smem_desc_sw128(smem_u32(sm.h[s]), kHalf, 1024);
#pragma unroll
            for (int kk = 0; kk < 8; ++kk)
              mma_ts(tmem + kColO, tmem + kColW + 64 * slot + 8 * kk, hd + (uint64_t)(kk * 2048 >> 4), idesc_h,
                     (n > 0 || kk > 0) ? 1u : 0u);
            mma_commit(&sm.bar_empty[slot]);
            ++n;
          }
        }
      }
      mma_commit(&sm.bar_final);
      mma_commit(&sm.bar_drain);
      const uint64_t t0 = globaltimer_ns();
      while (!mbar_try_wait(&sm.bar_drain, 0) && globaltimer_ns() - t0 < p.wait_ns) {}
    }
  } else {
    // ======================== W builders + epilogue ========================
    const unsigned FULL = 0xffffffffu;
    const int r = threadIdx.x;
    const uint32_t trow = tmem + ((uint32_t)(warp * 32) << 16);
    const bool upper = pair && r >= 64;
    const uint32_t* own = upper ? sm.bitsB : sm.bitsA;
    const int myq = upper ? qb : qa;
    const int rloc = pair ? (r & 63) : r;
    const bool row_valid = rloc < block_count(myq, p.L, p.block) && (!upper || has_b);
    const size_t grow_idx = (size_t)bh * p.L + (size_t)myq * p.block + rloc;
    float2 rs = make_float2(0.f, 0.f);
    if (row_valid) rs = p.rowstats[grow_idx];
    float* arow = sm.alpha + r * kAlphaStride;

    bool ok = __all_sync(FULL, wait_or_abort(sm, &sm.bar_q, 0, p));
    // this row of Q as 64 bf16 pairs (the tile is 128B-swizzled: 16-byte chunk c of a row sits at
    // chunk c ^ (row & 7))
    uint32_t q2[64];
#pragma unroll
    for (int hf = 0; hf < 2; ++hf) {
#pragma unroll
      for (int c = 0; c < 8; ++c) {
        const uint4 u = *reinterpret_cast<const uint4*>(sm.q + hf * kHalf + r * 128 + ((c ^ (r & 7)) << 4));
        q2[hf * 32 + 4 * c] = u.x;
        q2[hf * 32 + 4 * c + 1] = u.y;
        q2[hf * 32 + 4 * c + 2] = u.z;
        q2[hf * 32 + 4 * c + 3] = u.w;
      }
    }
    int n = 0;
    for (int ct = 0; ct < nct && ok; ++ct) {
      ok = __all_sync(FULL, wait_or_abort(sm, &sm.bar_cfull, ct & 1, p));
      if (!ok) break;
      tc_fence_after();
      for (int ch = 0; ch < 4 && ok; ++ch) {
        const int w = 4 * ct + ch;
        const uint32_t pm = proc_word(sm, w, p.nb);
        if (pm == 0) continue;
        float c[32];
        tmem_ld32(trow + kColC + 32 * ch, c);
        tmem_ld_wait();
        const uint32_t am = row_valid ? (pm & ~own[w]) : 0u;
#pragma unroll
        for (int x = 0; x < 32; ++x)
          arow[x] = ((am >> x) & 1u) ? ex2(fmaf(c[x], p.scale_log2, -rs.x)) * rs.y : 0.f;
        for (uint32_t mm = pm; mm; mm &= mm - 1) {
          const int x = __ffs(mm) - 1, slot = n % kR;
          if (n >= kR) {
            ok = __all_sync(FULL, wait_or_abort(sm, &sm.bar_empty[slot], ((n / kR) - 1) & 1, p));
            if (!ok) break;
            tc_fence_after();
          }
          const float a = arow[x];
          const uint32_t a2 = pack_bf16x2(a, a);
          uint32_t wv[64];
#pragma unroll
          for (int i = 0; i < 64; ++i) wv[i] = mul_bf16x2(q2[i], a2);
          tmem_st32(trow + kColW + 64 * slot, reinterpret_cast<const float*>(wv));
          tmem_st32(trow + kColW + 64 * slot + 32, reinterpret_cast<const float*>(wv + 32));
          tmem_st_wait();
          tc_fence_before();
          mbar_arrive(&sm.bar_full[slot]);
          ++n;
        }
      }
      if (!ok) break;
      tc_fence_before();
      mbar_arrive(&sm.bar_cempty);
    }
    if (ok) ok = __all_sync(FULL, wait_or_abort(sm, &sm.bar_final, 0, p));
    if (ok) {
      tc_fence_after();
#pragma unroll
      for (int ch = 0; ch < 4; ++ch) {
        float ov[32];
        tmem_ld32(trow + kColO + 32 * ch, ov);
        tmem_ld_wait();
        if (row_valid) store_row32(p, grow_idx, ch, ov);
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  __syncwarp();
  if (warp == 5) tmem_dealloc(tmem, kTmemCols);
}

}  // namespace

cudaError_t launch_perblock_sm100(const Dims& g, const AttnMaps& maps, const CUtensorMap& hdiff,
                                  const int32_t* sel, const int32_t* order, int keep_k, const float2* rowstats,
                                  const float* o32, void* o, int* status, unsigned long long wait_ns,
                                  cudaStream_t stream) {
  Params p;
  p.L = g.L;
  p.nb = g.nb;
  p.block = g.block;
  p.keep_k = keep_k;
  p.scale_log2 = g.scale * 1.4426950408889634f;
  p.sel = sel;
  p.order = order;
  p.rowstats = rowstats;
  p.o32 = o32;
  p.o = static_cast<__nv_bfloat16*>(o);
  p.status = status;
  p.wait_ns = wait_ns;
  const size_t smem = sizeof(Smem) + 1024;
  cudaError_t e;
  if ((e = set_max_dynamic_smem(reinterpret_cast<const void*>(perblock_sm100), smem))) return e;
  const int ntiles = g.block == 64 ? (g.nb + 1) / 2 : g.nb;
  perblock_sm100<<<dim3(ntiles, g.BH()), kThreads, smem, stream>>>(maps, hdiff, p);
  return cudaGetLastError();
}

}  // namespace pisa
