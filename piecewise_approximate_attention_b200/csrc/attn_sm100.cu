// Fused exact-or-approximate attention for sm_100a: TMA + tcgen05 (TMEM accumulators).
//
// "PISA: Piecewise Sparse Attention Is Wiser for Efficient Diffusion Transformers", §2 방법론,
// 하드웨어 구현: one FlashAttention-style online softmax interleaves
//   stage 1  exact attention over the selected key blocks S_i (loaded to on-chip memory),
//   stage 2  the zeroth-order scan of the unselected blocks: logits q_t . kbar_j against the block
//            centroids and values sum_n v_n, with denominator weight cnt_j,
//   stage 3  the global first-order correction s (q_t Hbar) sum_{j in U_i} alpha_tj, injected before
//            the division o_t = N_t / D_t.
//
// Mapping onto B200 (one CTA = one 128-row query tile; two CTAs share an SM):
//   * Q tile 128 x 128 bf16 in shared memory (two 64-column 128B-swizzled halves, filled by TMA).
//     With 64-token blocks a tile holds two query blocks a, b (consecutive entries of the router's
//     pairing order); with 128-token blocks it holds one.
//   * The tile walks a list of 128-row "key tiles": first the union of S_a and S_b (two 64-token key
//     blocks per tile, each half masked for the query block that did not select it), then, in PISA
//     mode, ceil(nb/128) centroid tiles (kbar_j as keys, vsum_j as values; columns of selected blocks
//     masked).  Both kinds run through the same tcgen05 MMAs: S = Q K^T into TMEM (fp32), softmax in
//     registers (one thread per row), P (fp16) written back over S in TMEM, O += P V with P read from
//     TMEM and V from shared memory (MN-major).
//   * kF8 (PISA_BF16_FP8QK): Q, K and the centroids come as e4m3 copies and S is a kind::f8f6f4
//     product (K = 32 per instruction); each half's raw scores are scaled by the row's q scale times
//     the key block's (or centroid tile's) k scale.  The correction keeps the bf16 Q tile.
//   * P enters the PV product in fp16 (11 significant bits) against an fp16 copy of the values
//     (v / vscale, a per-head power of two, written by the pre-computation).  That precision lets
//     the running max lag the true row max by up to 2^8 (weights up to 256), so O is rescaled in
//     TMEM only when a row max jumps by more than that; with bf16 weights the lag measured ~10x
//     larger errors on rows dominated by one key.  The epilogue multiplies O back by vscale.
//   * The correction is one more MMA, Q (s Hbar^T), into the S columns after the last PV; the
//     epilogue computes o = (O + A * (Q s Hbar)) / l with A = sum of alpha over U_i.
// Warp roles: warps 0-3 softmax + epilogue (TMEM lanes 0-127), warp 4 TMA producer, warp 5 MMA
// issuer and TMEM owner.  Every mbarrier wait is bounded; a timeout sets the status word and the
// CTA drains its own in-flight work, frees TMEM and exits.
#include <cuda.h>

#include "common.cuh"
#include "sm100.cuh"

namespace pisa {
namespace {
using namespace sm100;

constexpr int D = 128;
constexpr int kThreads = 192;
constexpr int kHalf = 128 * 64 * 2;        // one 128-row x 64-column bf16 half: 16 KB
constexpr int kTileBytes = 2 * kHalf;      // 32 KB
constexpr uint32_t kTmemCols = 256;
constexpr uint32_t kColS = 0, kColO = 128;   // S/P of the two 64-key halves at 0 and 64, O at 128
constexpr int kWords = 128;                // selection bitmap words (nb <= 4096)
constexpr float kLazyLog2 = 8.f;           // the running max may lag by 2^8 (fp16 weights up to 256)
#ifndef PISA_ATTN_KSTAGES
#define PISA_ATTN_KSTAGES 1
#endif
#ifndef PISA_ATTN_VSTAGES
#define PISA_ATTN_VSTAGES 1
#endif
constexpr int kKS = PISA_ATTN_KSTAGES;     // key-tile buffers in shared memory
constexpr int kVS = PISA_ATTN_VSTAGES;     // value-tile buffers

struct alignas(1024) Smem {
  uint8_t v[kVS][kTileBytes];
  uint8_t q[kTileBytes];
  uint8_t k[kKS][kTileBytes];
  uint64_t bar_kfull[kKS], bar_kempty[kKS], bar_vfull[kVS], bar_vempty[kVS];
  uint64_t bar_sfull[2], bar_pfull[2], bar_odone[2];
  uint64_t bar_q, bar_final, bar_drain;
  uint64_t bar_q16;          // e4m3 logits: the bf16 Q tile for the correction, loaded at the end
  uint32_t tmem_base;
  int abort;
  int n_exact, n_cent, need_corr;
  uint32_t bitsA[kWords];
  uint32_t bitsB[kWords];
};

struct Params {
  int L, nb, block, keep_k, mode, dense;
  float scale_log2;
  float lazy;                // rescale O only when the row max grows by more than this (logit units)
  const float* vscale;       // [B*H] value scale of the fp16 value operands
  int fault;                 // test-only fault injection (pisa_testing.h); 0 in normal calls
  const int32_t* sel;
  const int32_t* order;
  const float* qscale;       // e4m3 logits only: per-row, per-key-block and per-centroid-tile scales
  const float* kscale;
  const float* kbscale;
  __nv_bfloat16* o;
  float2* rowstats;          // nullable [B*H][L]: (softmax offset m*s*log2(e), 1/D_t) per row
  float* o32;                // nullable [B*H][L][D]: the output in fp32 instead of bf16 in o
  int* status;
  unsigned long long wait_ns;
};

__device__ __forceinline__ bool bit_of(const uint32_t* bits, int j) { return (bits[j >> 5] >> (j & 31)) & 1u; }

// Ascending enumeration of the key blocks in S_a | S_b.  The producer and every softmax thread run
// identical copies, so the key-tile sequence needs no hand-off between roles.
struct UnionIter {
  int w = 0;
  uint32_t cur = 0;
  __device__ __forceinline__ int next(const uint32_t* a, const uint32_t* b) {
    while (cur == 0) {
      if (w >= kWords) return -1;
      cur = a[w] | b[w];
      ++w;
    }
    const int j = (w - 1) * 32 + __ffs(cur) - 1;
    cur &= cur - 1;
    return j;
  }
};

// Key tile t: kind 0 = exact (key blocks j0, j1; j1 = -1 when absent or block == 128),
// kind 1 = centroid tile starting at centroid j0.
struct KeyTile {
  int kind, j0, j1;
};
__device__ __forceinline__ KeyTile key_tile(int t, int n_exact, bool pair, UnionIter& it, const uint32_t* a,
                                            const uint32_t* b) {
  KeyTile kt;
  if (t < n_exact) {
    kt.kind = 0;
    kt.j0 = it.next(a, b);
    kt.j1 = pair ? it.next(a, b) : -1;
  } else {
    kt.kind = 1;
    kt.j0 = (t - n_exact) * 128;
    kt.j1 = -1;
  }
  return kt;
}

__device__ __forceinline__ bool wait_or_abort(Smem& sm, uint64_t* bar, uint32_t parity, const Params& p) {
  if (mbar_wait_bounded(bar, parity, &sm.abort, p.wait_ns)) return true;
  *reinterpret_cast<volatile int*>(&sm.abort) = 1;
  set_status(p.status, PISA_DEVERR_WAIT_TIMEOUT);
  return false;
}

// Fills the selection bitmap of query block `qi` (validating entries) — all threads of the CTA.
__device__ void build_bits(uint32_t* bits, const Params& p, int bh, int qi) {
  if (p.dense) {
    for (int w = threadIdx.x; w < kWords; w += kThreads) {
      const int lo = w * 32;
      bits[w] = lo >= p.nb ? 0u : (p.nb - lo >= 32 ? 0xffffffffu : ((1u << (p.nb - lo)) - 1u));
    }
    return;
  }
  const int32_t* row = p.sel + ((size_t)bh * p.nb + qi) * p.keep_k;
  for (int e = threadIdx.x; e < p.keep_k; e += kThreads) {
    const int j = row[e];
    bool ok = j >= 0 && j < p.nb;
    if (e > 0 && row[e - 1] >= j) set_status(p.status, PISA_DEVERR_BAD_SELECTION);
    if (!ok) {
      set_status(p.status, PISA_DEVERR_BAD_SELECTION);
      continue;
    }
    const uint32_t old = atomicOr(&bits[j >> 5], 1u << (j & 31));
    if (old & (1u << (j & 31))) set_status(p.status, PISA_DEVERR_BAD_SELECTION);
  }
}

// kF8: logits from e4m3 copies of q, k and kbar (kind::f8f6f4 MMAs, K = 32 per instruction); each
// half's raw scores are scaled by its row's q scale times the key block's (or centroid tile's) k
// scale before they enter the max and the exponent.  The correction keeps the bf16 Q tile.
template <bool kF8>
__global__ void __launch_bounds__(kThreads, 2)
attn_sm100(const __grid_constant__ AttnMaps maps, const Params p) {
  extern __shared__ uint8_t smem_raw[];
  Smem& sm = *reinterpret_cast<Smem*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int tile = blockIdx.x, bh = blockIdx.y;
  const bool pair = p.block == 64;

  // ---- query blocks of this tile ----
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
  if (qa < 0 || qa >= p.nb || qb < 0 || qb >= p.nb) {
    if (threadIdx.x == 0) set_status(p.status, PISA_DEVERR_BAD_SELECTION);
    return;
  }

  // ---- set-up: barriers, TMEM, selection bitmaps ----
  for (int w = threadIdx.x; w < kWords; w += kThreads) { sm.bitsA[w] = 0u; sm.bitsB[w] = 0u; }
  if (threadIdx.x == 0) {
    mbar_init(&sm.bar_q, 1);
    for (int i = 0; i < kKS; ++i) {
      mbar_init(&sm.bar_kfull[i], 1);
      mbar_init(&sm.bar_kempty[i], 1);
    }
    for (int i = 0; i < kVS; ++i) {
      mbar_init(&sm.bar_vfull[i], 1);
      mbar_init(&sm.bar_vempty[i], 1);
    }
    for (int hh = 0; hh < 2; ++hh) {
      mbar_init(&sm.bar_sfull[hh], 1);
      mbar_init(&sm.bar_pfull[hh], 128);
      mbar_init(&sm.bar_odone[hh], 1);
    }
    mbar_init(&sm.bar_final, 1);
    mbar_init(&sm.bar_drain, 1);
    mbar_init(&sm.bar_q16, 1);
    sm.abort = 0;
    fence_mbar_init();
  }
  if (warp == 5) {
    tmem_alloc(&sm.tmem_base, kTmemCols);
    tmem_relinquish();
  }
  __syncthreads();
  build_bits(sm.bitsA, p, bh, qa);
  if (has_b) build_bits(sm.bitsB, p, bh, qb);
  __syncthreads();
  if (!has_b)
    for (int w = threadIdx.x; w < kWords; w += kThreads) sm.bitsB[w] = sm.bitsA[w];
  if (warp == 0) {
    int cnt = 0;
    for (int w = lane; w < kWords; w += 32) cnt += __popc(sm.bitsA[w] | sm.bitsB[w]);
    for (int o = 16; o > 0; o >>= 1) cnt += __shfl_xor_sync(0xffffffffu, cnt, o);
    if (lane == 0) {
      sm.n_exact = pair ? (cnt + 1) / 2 : cnt;
      const bool approx = p.mode == PISA_MODE_PISA && !p.dense && p.keep_k < p.nb;
      sm.n_cent = approx ? (p.nb + 127) / 128 : 0;
      sm.need_corr = approx ? 1 : 0;
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = sm.tmem_base;
  const int n_exact = sm.n_exact, T = sm.n_exact + sm.n_cent;
  const bool need_corr = sm.need_corr != 0;

  if (warp == 4) {
    // =============================== TMA producer ===============================
    if (lane == 0) {
      tma_prefetch_desc(&maps.q);
      tma_prefetch_desc(&maps.k);
      tma_prefetch_desc(&maps.v);
      const bool issued_q = p.fault != 1;   // fault 1 (tests only): never load Q, so the MMA warp's wait runs out
      if (issued_q) {
        if (kF8) {             // e4m3 Q: one 128-byte row per token, 16 KB
          mbar_expect_tx(&sm.bar_q, kHalf);
          tma_load_3d(sm.q, &maps.q8, &sm.bar_q, 0, qa * p.block, bh);
          if (pair) tma_load_3d(sm.q + 64 * 128, &maps.q8, &sm.bar_q, 0, qb * p.block, bh);
        } else {
          mbar_expect_tx(&sm.bar_q, kTileBytes);
          tma_load_3d(sm.q, &maps.q, &sm.bar_q, 0, qa * p.block, bh);
          tma_load_3d(sm.q + kHalf, &maps.q, &sm.bar_q, 64, qa * p.block, bh);
          if (pair) {
            tma_load_3d(sm.q + 64 * 128, &maps.q, &sm.bar_q, 0, qb * p.block, bh);
            tma_load_3d(sm.q + kHalf + 64 * 128, &maps.q, &sm.bar_q, 64, qb * p.block, bh);
          }
        }
      }
      UnionIter it;
      int issued_k = 0, issued_v = 0, issued_q16 = 0;
      bool ok = true;
      for (int t = 0; t < T && ok; ++t) {
        const int ks = t % kKS, vs = t % kVS;
        if (t >= kKS && !(ok = wait_or_abort(sm, &sm.bar_kempty[ks], ((t / kKS) - 1) & 1, p))) break;
        const KeyTile kt = key_tile(t, n_exact, pair, it, sm.bitsA, sm.bitsB);
        const int j1 = kt.j1 >= 0 ? kt.j1 : kt.j0;     // absent second block: reload the first, masked
        uint8_t* kb = sm.k[ks];
        uint64_t* kf = &sm.bar_kfull[ks];
        if (kF8) {               // e4m3 keys or centroids: 128 rows of 128 bytes
          mbar_expect_tx(kf, kHalf);
          if (kt.kind == 0) {
            if (pair) {
              tma_load_3d(kb, &maps.k8, kf, 0, kt.j0 * 64, bh);
              tma_load_3d(kb + 64 * 128, &maps.k8, kf, 0, j1 * 64, bh);
            } else {
              tma_load_3d(kb, &maps.k8, kf, 0, kt.j0 * 128, bh);
            }
          } else {
            tma_load_3d(kb, &maps.kbar8, kf, 0, kt.j0, bh);
          }
        } else {
          mbar_expect_tx(kf, kTileBytes);
          if (kt.kind == 0) {
            if (pair) {
              tma_load_3d(kb, &maps.k, kf, 0, kt.j0 * 64, bh);
              tma_load_3d(kb + kHalf, &maps.k, kf, 64, kt.j0 * 64, bh);
              tma_load_3d(kb + 64 * 128, &maps.k, kf, 0, j1 * 64, bh);
              tma_load_3d(kb + kHalf + 64 * 128, &maps.k, kf, 64, j1 * 64, bh);
            } else {
              tma_load_3d(kb, &maps.k, kf, 0, kt.j0 * 128, bh);
              tma_load_3d(kb + kHalf, &maps.k, kf, 64, kt.j0 * 128, bh);
            }
          } else {
            tma_load_3d(kb, &maps.kbar, kf, 0, kt.j0, bh);
            tma_load_3d(kb + kHalf, &maps.kbar, kf, 64, kt.j0, bh);
          }
        }
        ++issued_k;
        if (t >= kVS && !(ok = wait_or_abort(sm, &sm.bar_vempty[vs], ((t / kVS) - 1) & 1, p))) break;
        uint8_t* vb = sm.v[vs];
        uint64_t* vf = &sm.bar_vfull[vs];
        mbar_expect_tx(vf, kTileBytes);
        if (kt.kind == 0) {
          if (pair) {
            tma_load_3d(vb, &maps.v, vf, 0, kt.j0 * 64, bh);
            tma_load_3d(vb + kHalf, &maps.v, vf, 64, kt.j0 * 64, bh);
            tma_load_3d(vb + 64 * 128, &maps.v, vf, 0, j1 * 64, bh);
            tma_load_3d(vb + kHalf + 64 * 128, &maps.v, vf, 64, j1 * 64, bh);
          } else {
            tma_load_3d(vb, &maps.v, vf, 0, kt.j0 * 128, bh);
            tma_load_3d(vb + kHalf, &maps.v, vf, 64, kt.j0 * 128, bh);
          }
        } else {
          tma_load_3d(vb, &maps.vsum, vf, 0, kt.j0, bh);
          tma_load_3d(vb + kHalf, &maps.vsum, vf, 64, kt.j0, bh);
        }
        ++issued_v;
      }
      if (ok && need_corr) {
        const int ks = T % kKS;
        if (T < kKS || (ok = wait_or_abort(sm, &sm.bar_kempty[ks], ((T / kKS) - 1) & 1, p))) {
          mbar_expect_tx(&sm.bar_kfull[ks], kTileBytes);
          tma_load_3d(sm.k[ks], &maps.hbar, &sm.bar_kfull[ks], 0, 0, bh);
          tma_load_3d(sm.k[ks] + kHalf, &maps.hbar, &sm.bar_kfull[ks], 64, 0, bh);
          ++issued_k;
        }
        if (kF8 && ok) {
          // the correction multiplies the bf16 Q tile: into the value buffer once the last PV is done
          const int vs = T % kVS;
          if (T < kVS || (ok = wait_or_abort(sm, &sm.bar_vempty[vs], ((T / kVS) - 1) & 1, p))) {
            mbar_expect_tx(&sm.bar_q16, kTileBytes);
            tma_load_3d(sm.v[vs], &maps.q, &sm.bar_q16, 0, qa * p.block, bh);
            tma_load_3d(sm.v[vs] + kHalf, &maps.q, &sm.bar_q16, 64, qa * p.block, bh);
            if (pair) {
              tma_load_3d(sm.v[vs] + 64 * 128, &maps.q, &sm.bar_q16, 0, qb * p.block, bh);
              tma_load_3d(sm.v[vs] + kHalf + 64 * 128, &maps.q, &sm.bar_q16, 64, qb * p.block, bh);
            }
            issued_q16 = 1;
          }
        }
      }
      {
        // drain: every copy issued must land before this CTA's shared memory is released (in a
        // normal run the MMA warp has waited for all of them, so these waits return at once).
        // Each wait has its own deadline, so one that gives up cannot cut the others short.
        if (issued_q) mbar_drain(&sm.bar_q, 0, p.wait_ns);
        if (issued_q16) mbar_drain(&sm.bar_q16, 0, p.wait_ns);
        for (int i = max(0, issued_k - kKS); i < issued_k; ++i) mbar_drain(&sm.bar_kfull[i % kKS], (i / kKS) & 1, p.wait_ns);
        for (int i = max(0, issued_v - kVS); i < issued_v; ++i) mbar_drain(&sm.bar_vfull[i % kVS], (i / kVS) & 1, p.wait_ns);
      }
    }
  } else if (warp == 5) {
    // =============================== MMA issuer ===============================
    // Each 128-key tile is two 64-key halves with their own S buffers, so the tensor core works on
    // one half while the softmax warps work on the other:
    //   S_a(0) S_b(0) | PV_a(0) S_a(1) PV_b(0) S_b(1) | PV_a(1) S_a(2) PV_b(1) S_b(2) | ...
    // PV_h(t) reads P_h(t) from the S_h columns; S_h(t+1) overwrites them afterwards, in issue order.
    if (lane == 0) {
      const uint32_t idesc_s = idesc_bf16_f32(128, 64, false, false);
      const uint32_t idesc_pv = idesc_f16_f32(128, 128, false, true);
      const uint32_t idesc_c = idesc_bf16_f32(128, 128, false, false);
      const uint64_t qd = smem_desc_sw128(smem_u32(sm.q), 16, 1024);
      bool ok = wait_or_abort(sm, &sm.bar_q, 0, p);
      tc_fence_after();
      // S_h(t) = Q K_h(t)^T into columns 64h (keys 64h..64h+63 of tile t)
      auto issue_s = [&](int t, int hh) -> bool {
        const int ks = t % kKS;
        if (hh == 0) {
          if (!wait_or_abort(sm, &sm.bar_kfull[ks], (t / kKS) & 1, p)) return false;
          tc_fence_after();
        }
        const uint64_t kd = smem_desc_sw128(smem_u32(sm.k[ks]) + 8192 * hh, 16, 1024);
        if (kF8) {
          // e4m3 rows are 128 bytes: the four K = 32 steps are 32-byte column offsets of one row
#pragma unroll
          for (int kk = 0; kk < 4; ++kk)
            mma_ss_f8(tmem + kColS + 64 * hh, qd + (kk * 32 >> 4), kd + (kk * 32 >> 4), idesc_e4m3_f32(128, 64), kk > 0);
        } else {
#pragma unroll
          for (int kk = 0; kk < 8; ++kk) {
            const uint32_t off = ((kk >> 2) * kHalf + (kk & 3) * 32) >> 4;   // start-address field units
            mma_ss(tmem + kColS + 64 * hh, qd + off, kd + off, idesc_s, kk > 0);
          }
        }
        mma_commit(&sm.bar_sfull[hh]);
        if (hh == 1) mma_commit(&sm.bar_kempty[ks]);
        return true;
      };
      // O += P_h(t) V_h(t): P from TMEM columns 64h.., V rows 64h..64h+63 (MN-major)
      auto issue_pv = [&](int t, int hh) -> bool {
        const int vs = t % kVS;
        if (!wait_or_abort(sm, &sm.bar_pfull[hh], t & 1, p)) return false;
        if (hh == 0 && !wait_or_abort(sm, &sm.bar_vfull[vs], (t / kVS) & 1, p)) return false;
        tc_fence_after();
        const uint64_t vd = smem_desc_sw128(smem_u32(sm.v[vs]) + 8192 * hh, kHalf, 1024);
#pragma unroll
        for (int kk = 0; kk < 4; ++kk)
          mma_ts(tmem + kColO, tmem + kColS + 64 * hh + kk * 8, vd + (uint64_t)(kk * 2048 >> 4), idesc_pv,
                 (t > 0 || hh > 0 || kk > 0) ? 1u : 0u);
        mma_commit(&sm.bar_odone[hh]);
        if (hh == 1) mma_commit(&sm.bar_vempty[vs]);
        return true;
      };
      if (ok && T > 0) ok = issue_s(0, 0) && issue_s(0, 1);
      for (int t = 0; t < T && ok; ++t) {
        ok = issue_pv(t, 0);
        if (ok && t + 1 < T) ok = issue_s(t + 1, 0);
        if (ok) ok = issue_pv(t, 1);
        if (ok && t + 1 < T) ok = issue_s(t + 1, 1);
      }
      if (ok && need_corr) {
        // Q (s Hbar^T) into columns 0..127, after every PV has read its P there
        const int ks = T % kKS;
        // with e4m3 logits the correction's A operand is the bf16 Q tile loaded into the value buffer
        if ((ok = wait_or_abort(sm, &sm.bar_kfull[ks], (T / kKS) & 1, p)) &&
            (!kF8 || (ok = wait_or_abort(sm, &sm.bar_q16, 0, p)))) {
          tc_fence_after();
          const uint64_t kd = smem_desc_sw128(smem_u32(sm.k[ks]), 16, 1024);
          const uint64_t ad = kF8 ? smem_desc_sw128(smem_u32(sm.v[T % kVS]), 16, 1024) : qd;
#pragma unroll
          for (int kk = 0; kk < 8; ++kk) {
            const uint32_t off = ((kk >> 2) * kHalf + (kk & 3) * 32) >> 4;
            mma_ss(tmem + kColS, ad + off, kd + off, idesc_c, kk > 0);
          }
        }
      }
      mma_commit(&sm.bar_final);
      // every MMA issued above has completed once bar_drain flips (bounded)
      mma_commit(&sm.bar_drain);
      const uint64_t t0 = globaltimer_ns();
      while (!mbar_try_wait(&sm.bar_drain, 0) && globaltimer_ns() - t0 < p.wait_ns) {}
    }
  } else {
    // =========================== softmax + epilogue ===========================
    // Thread r owns tile row r (TMEM lane r) and walks the 64-key halves in MMA order.  Decisions
    // that guard .sync.aligned TMEM accesses are made warp-uniform.
    const unsigned FULL = 0xffffffffu;
    const int r = threadIdx.x;
    const uint32_t trow = tmem + ((uint32_t)(warp * 32) << 16);
    const bool upper = pair && r >= 64;
    const uint32_t* bits = upper ? sm.bitsB : sm.bitsA;
    const int myq = upper ? qb : qa;
    const int rloc = pair ? (r & 63) : r;
    const bool row_valid = rloc < block_count(myq, p.L, p.block) && (!upper || has_b);
    const float last_cnt = (float)block_count(p.nb - 1, p.L, p.block);
    float m = -INFINITY, l = 0.f, A = 0.f;
    // e4m3 logits: this row's q scale, and the k scales of the current tile's two halves
    const float qsc = (kF8 && row_valid) ? p.qscale[(size_t)bh * p.L + (size_t)myq * p.block + rloc] : 1.f;
    float ksc0 = 1.f, ksc1 = 1.f;
    UnionIter it;
    KeyTile kt{0, 0, -1};
    bool ok = true;
    for (int u = 0; u < 2 * T; ++u) {
      const int t = u >> 1, hh = u & 1;
      if (hh == 0) {
        kt = key_tile(t, n_exact, pair, it, sm.bitsA, sm.bitsB);
        if (kF8) {   // issued before the wait, so the loads overlap it
          const size_t kb0 = (size_t)bh * p.nb;
          if (kt.kind == 1) {
            ksc0 = ksc1 = p.kbscale[(size_t)bh * ((p.nb + 127) / 128) + (kt.j0 >> 7)];
          } else {
            ksc0 = p.kscale[kb0 + kt.j0];
            ksc1 = pair ? (kt.j1 >= 0 ? p.kscale[kb0 + kt.j1] : 1.f) : ksc0;
          }
        }
      }
      const bool centroid = kt.kind == 1;
      // validity of this half's 64 columns for this row's query block, 32 per word (warp-uniform:
      // a warp's rows belong to one query block)
      uint32_t vm0, vm1;
      if (!centroid) {
        const int jh = pair ? (hh ? kt.j1 : kt.j0) : kt.j0;
        const int cnt = (jh >= 0 && bit_of(bits, jh)) ? block_count(jh, p.L, p.block) : 0;
        const int r0 = cnt - (pair ? 0 : 64 * hh), r1 = r0 - 32;   // valid columns left in each word
        vm0 = r0 >= 32 ? FULL : (r0 > 0 ? ((1u << r0) - 1u) : 0u);
        vm1 = r1 >= 32 ? FULL : (r1 > 0 ? ((1u << r1) - 1u) : 0u);
      } else {
        const int j0 = kt.j0 + 64 * hh, w0 = j0 >> 5;
        const int r0 = p.nb - j0, r1 = r0 - 32;
        vm0 = (r0 >= 32 ? FULL : (r0 > 0 ? ((1u << r0) - 1u) : 0u)) & ~(w0 < kWords ? bits[w0] : 0u);
        vm1 = (r1 >= 32 ? FULL : (r1 > 0 ? ((1u << r1) - 1u) : 0u)) & ~(w0 + 1 < kWords ? bits[w0 + 1] : 0u);
      }
      ok = __all_sync(FULL, wait_or_abort(sm, &sm.bar_sfull[hh], t & 1, p));
      if (!ok) break;
      tc_fence_after();
      if (__all_sync(FULL, (vm0 | vm1) == 0u)) {
        // Every column masked for this warp's rows (in a paired tile, a key block that only the other
        // query block selected): all weights are exactly 0 and m, l, A stay as they are, so the scores
        // are not read and only P = 0 is written for the PV product.
        uint32_t zero[16];
#pragma unroll
        for (int x = 0; x < 16; ++x) zero[x] = 0u;
        tmem_st16(trow + kColS + 64 * hh, zero);
        tmem_st16(trow + kColS + 64 * hh + 16, zero);
        tmem_st_wait();
        tc_fence_before();
        mbar_arrive(&sm.bar_pfull[hh]);
        continue;
      }
      const float sl = kF8 ? qsc * (hh ? ksc1 : ksc0) : 1.f;   // raw MMA score -> logit
      float s[64];
      tmem_ld32(trow + kColS + 64 * hh, s);
      tmem_ld32(trow + kColS + 64 * hh + 32, s + 32);
      tmem_ld_wait();
      if (vm0 != FULL) {
#pragma unroll
        for (int x = 0; x < 32; ++x) s[x] = ((vm0 >> x) & 1u) ? s[x] : -INFINITY;
      }
      if (vm1 != FULL) {
#pragma unroll
        for (int x = 0; x < 32; ++x) s[32 + x] = ((vm1 >> x) & 1u) ? s[32 + x] : -INFINITY;
      }
      float t0 = fmaxf(s[0], s[1]), t1 = fmaxf(s[2], s[3]), t2 = fmaxf(s[4], s[5]), t3 = fmaxf(s[6], s[7]);
#pragma unroll
      for (int c = 8; c < 64; c += 8) {
        t0 = fmax3(t0, s[c], s[c + 1]);
        t1 = fmax3(t1, s[c + 2], s[c + 3]);
        t2 = fmax3(t2, s[c + 4], s[c + 5]);
        t3 = fmax3(t3, s[c + 6], s[c + 7]);
      }
      const float hmax = fmaxf(fmaxf(t0, t1), fmaxf(t2, t3));
      const float m_new = fmaxf(m, kF8 ? hmax * sl : hmax);   // logit units
      const bool grow = m_new > m + p.lazy;
      const float f = grow ? ex2((m - m_new) * p.scale_log2) : 1.f;   // 0 when m = -inf
      if (grow) {
        l *= f;
        A *= f;
        m = m_new;
      }
      float slast = -INFINITY;     // raw logit of the last (short) key block, when this half holds it
      const int cl = p.nb - 1 - kt.j0 - 64 * hh;
      const bool has_last = centroid && cl >= 0 && cl < 64 && last_cnt != (float)p.block;
      if (has_last) {
#pragma unroll
        for (int c = 0; c < 64; ++c) slast = c == cl ? s[c] : slast;
      }
      // p = 2^(s*scale*log2e - m*scale*log2e) (masked entries are -inf and give exactly 0), two at a
      // time with f32x2 arithmetic; P (fp16 pairs) goes over the first 32 columns of this half's S
      const float mb = m == -INFINITY ? 0.f : m * p.scale_log2;
      const float scl = kF8 ? p.scale_log2 * sl : p.scale_log2;
      const uint64_t sc2 = f2_pack(scl, scl), nmb2 = f2_pack(-mb, -mb);
      uint64_t acc2 = f2_pack(0.f, 0.f);
#pragma unroll
      for (int ch = 0; ch < 2; ++ch) {
        uint32_t pk[16];
#pragma unroll
        for (int x = 0; x < 32; x += 2) {
          const int c = 32 * ch + x;
          float x0, x1;
          f2_unpack(f2_fma(f2_pack(s[c], s[c + 1]), sc2, nmb2), x0, x1);
          const float p0 = ex2(x0), p1 = ex2(x1);
          acc2 = f2_add(acc2, f2_pack(p0, p1));
          pk[x >> 1] = pack_f16x2(p0, p1);
        }
        tmem_st16(trow + kColS + 64 * hh + 16 * ch, pk);
      }
      float ls0, ls1;
      f2_unpack(acc2, ls0, ls1);
      const float ls = ls0 + ls1;
      if (centroid) {
        // alpha of every unselected block enters D with weight cnt_j: `block` except the last one
        A += ls;
        l = fmaf((float)p.block, ls, l);
        if (has_last) l = fmaf(last_cnt - (float)p.block, ex2(fmaf(slast, scl, -mb)), l);
      } else {
        l += ls;
      }
      // O holds the PV products of the earlier halves; rescale it before PV of this half is released.
      // The previous half's PV was issued when its P was ready, long before this half's P was
      // computed, so the wait below is normally already satisfied.
      if (__any_sync(FULL, grow) && u > 0) {
        const int ph = hh ^ 1, pt = hh ? t : t - 1;
        ok = __all_sync(FULL, wait_or_abort(sm, &sm.bar_odone[ph], pt & 1, p));
        if (!ok) break;
        tc_fence_after();
#pragma unroll
        for (int ch = 0; ch < 4; ++ch) {
          float ov[32];
          tmem_ld32(trow + kColO + 32 * ch, ov);
          tmem_ld_wait();
#pragma unroll
          for (int x = 0; x < 32; ++x) ov[x] *= f;
          tmem_st32(trow + kColO + 32 * ch, ov);
        }
      }
      tmem_st_wait();
      tc_fence_before();
      mbar_arrive(&sm.bar_pfull[hh]);
    }
    if (ok) ok = __all_sync(FULL, wait_or_abort(sm, &sm.bar_final, 0, p));
    if (ok) {
      tc_fence_after();
      const float inv = 1.f / l, vsc = p.vscale[bh];
      const size_t grow_idx = (size_t)bh * p.L + (size_t)myq * p.block + rloc;
      __nv_bfloat16* orow = p.o + grow_idx * D;
      if (p.rowstats && row_valid) p.rowstats[grow_idx] = make_float2(m == -INFINITY ? 0.f : m * p.scale_log2, inv);
#pragma unroll
      for (int ch = 0; ch < 4; ++ch) {
        float ov[32], cv[32];
        tmem_ld32(trow + kColO + 32 * ch, ov);
        if (need_corr) tmem_ld32(trow + kColS + 32 * ch, cv);
        tmem_ld_wait();
        uint32_t pk[16];
#pragma unroll
        for (int x = 0; x < 32; x += 2) {
          float a = ov[x] * vsc, b = ov[x + 1] * vsc;
          if (need_corr) {
            a = fmaf(A, cv[x], a);
            b = fmaf(A, cv[x + 1], b);
          }
          pk[x >> 1] = pack_bf16x2(a * inv, b * inv);
        }
        if (row_valid && !p.o32) {
          uint4* dst = reinterpret_cast<uint4*>(orow + 32 * ch);
#pragma unroll
          for (int x = 0; x < 4; ++x) dst[x] = make_uint4(pk[4 * x], pk[4 * x + 1], pk[4 * x + 2], pk[4 * x + 3]);
        }
        if (row_valid && p.o32) {
          float4* dst = reinterpret_cast<float4*>(p.o32 + grow_idx * D + 32 * ch);
#pragma unroll
          for (int x = 0; x < 32; x += 4) {
            float a0 = ov[x] * vsc, a1 = ov[x + 1] * vsc, a2 = ov[x + 2] * vsc, a3 = ov[x + 3] * vsc;
            if (need_corr) {
              a0 = fmaf(A, cv[x], a0);
              a1 = fmaf(A, cv[x + 1], a1);
              a2 = fmaf(A, cv[x + 2], a2);
              a3 = fmaf(A, cv[x + 3], a3);
            }
            dst[x >> 2] = make_float4(a0 * inv, a1 * inv, a2 * inv, a3 * inv);
          }
        }
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

size_t attention_sm100_smem_bytes() { return sizeof(Smem) + 1024; }

cudaError_t launch_attention_sm100(const Dims& g, const AttnMaps& maps, const int32_t* sel, const int32_t* order,
                                   int keep_k, int mode, const float* vscale, const F8Scales& f8, void* o,
                                   float2* rowstats, float* o32, int* status, unsigned long long wait_ns, int fault,
                                   cudaStream_t stream) {
  Params p;
  p.L = g.L;
  p.nb = g.nb;
  p.block = g.block;
  p.keep_k = keep_k;
  p.mode = mode;
  p.dense = keep_k == g.nb;
  p.scale_log2 = g.scale * 1.4426950408889634f;
  p.lazy = kLazyLog2 / p.scale_log2;
  p.vscale = vscale;
  p.fault = fault;
  p.sel = sel;
  p.order = order;
  p.qscale = f8.q;
  p.kscale = f8.k;
  p.kbscale = f8.kb;
  p.o = static_cast<__nv_bfloat16*>(o);
  p.rowstats = rowstats;
  p.o32 = o32;
  p.status = status;
  p.wait_ns = wait_ns;
  const size_t smem = attention_sm100_smem_bytes();
  cudaError_t e;
  const int ntiles = g.block == 64 ? (g.nb + 1) / 2 : g.nb;
  const dim3 grid(ntiles, g.BH());
  if (f8.q) {
    if ((e = set_max_dynamic_smem(reinterpret_cast<const void*>(attn_sm100<true>), smem))) return e;
    attn_sm100<true><<<grid, kThreads, smem, stream>>>(maps, p);
  } else {
    if ((e = set_max_dynamic_smem(reinterpret_cast<const void*>(attn_sm100<false>), smem))) return e;
    attn_sm100<false><<<grid, kThreads, smem, stream>>>(maps, p);
  }
  return cudaGetLastError();
}

}  // namespace pisa
