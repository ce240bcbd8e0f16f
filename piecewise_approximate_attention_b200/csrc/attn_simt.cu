// Exact-or-approximate attention with fp32 FMA arithmetic (one thread per query row).
//
// "PISA: Piecewise Sparse Attention Is Wiser for Efficient Diffusion Transformers", §2 방법론:
// o_t = N_t / D_t with, for query t in block i,
//   N_t = sum_{j in S_i} sum_n e^{s q_t.k_n} v_n + sum_{j in U_i} alpha_tj vsum_j + s (q_t Hbar) sum_{U_i} alpha_tj
//   D_t = sum_{j in S_i} sum_n e^{s q_t.k_n}     + sum_{j in U_i} cnt_j alpha_tj,   alpha_tj = e^{s q_t.kbar_j}
// evaluated as one online softmax (running max m, all terms scaled by e^{-m}) over three stages
// (하드웨어 구현): exact tiles of the selected blocks, the zeroth-order scan over centroid tiles
// of the unselected blocks, then the first-order correction before normalisation.
// Serves fp32 inputs (the fp32-accurate mode).
#include "common.cuh"

namespace pisa {
namespace {

constexpr int kTile = 64;          // keys (or centroids) per shared-memory tile
constexpr int kMaxWords = 128;     // selection bitmap words: nb <= 4096

template <int D>
struct Smem {
  float q[128][D + 1];             // query rows (+1 pad: conflict-free per-thread rows)
  float kt[kTile][D];              // key / centroid tile (broadcast reads)
  float vt[kTile][D];              // value / value-sum tile
  float s[128][kTile + 1];         // per-thread scores of the current tile
  float w[kTile];                  // denominator weight of each tile column (1 or cnt_j)
  uint32_t selbits[kMaxWords];     // S_i as a bitmap over key blocks
  int32_t list[kMaxWords * 32];    // S_i as validated ascending list
  int nsel;
};

template <typename T, int D>
__global__ void __launch_bounds__(128) attn_simt(const T* __restrict__ q, const T* __restrict__ k,
                                                 const T* __restrict__ v, pisa_stats st,
                                                 const int32_t* __restrict__ sel, int keep_k, int mode, int L,
                                                 int block, int nb, float scale, T* __restrict__ o,
                                                 int* status) {
  extern __shared__ __align__(16) unsigned char raw[];
  Smem<D>& sm = *reinterpret_cast<Smem<D>*>(raw);
  const int i = blockIdx.x, bh = blockIdx.y, t = threadIdx.x;
  const int qs0 = i * block, qcnt = block_count(i, L, block);
  const size_t hoff = (size_t)bh * L * D;

  // selection list of this query block, validated (ascending, in range) and as a bitmap
  for (int w = t; w < kMaxWords; w += blockDim.x) sm.selbits[w] = 0u;
  __syncthreads();
  if (t == 0) {
    const int32_t* srow = sel + ((size_t)bh * nb + i) * keep_k;
    int n = 0, prev = -1;
    for (int e = 0; e < keep_k; ++e) {
      const int j = srow[e];
      if (j <= prev || j >= nb) { set_status(status, PISA_DEVERR_BAD_SELECTION); continue; }
      sm.list[n++] = j;
      sm.selbits[j >> 5] |= 1u << (j & 31);
      prev = j;
    }
    sm.nsel = n;
  }
  for (int idx = t; idx < qcnt * D; idx += blockDim.x) sm.q[idx / D][idx % D] = to_f32(q[hoff + (size_t)qs0 * D + idx]);
  __syncthreads();

  const bool row_ok = t < qcnt;
  float acc[D];
#pragma unroll
  for (int c = 0; c < D; ++c) acc[c] = 0.f;
  float m = -INFINITY, l = 0.f, A = 0.f;

  // one tile: columns [0, ncols) of sm.kt/sm.vt; valid(c) says whether the column counts;
  // centroid = true adds to A and weights the denominator by sm.w.
  auto process_tile = [&](int ncols, bool centroid, const bool* mask) {
    float tmax = -INFINITY;
    if (row_ok) {
      for (int c = 0; c < ncols; ++c) {
        float dot = 0.f;
#pragma unroll 16
        for (int a = 0; a < D; ++a) dot = fmaf(sm.q[t][a], sm.kt[c][a], dot);
        const float sv = mask[c] ? scale * dot : -INFINITY;
        sm.s[t][c] = sv;
        tmax = fmaxf(tmax, sv);
      }
      if (tmax > -INFINITY) {
        const float mn = fmaxf(m, tmax);
        const float corr = expf(m - mn);      // m = -inf on the first tile gives corr = 0
        l *= corr;
        A *= corr;
#pragma unroll
        for (int c = 0; c < D; ++c) acc[c] *= corr;
        m = mn;
        for (int c = 0; c < ncols; ++c) {
          const float p = expf(sm.s[t][c] - m);     // exp(-inf) = 0 for masked columns
          l = fmaf(centroid ? sm.w[c] : 1.f, p, l);
          if (centroid) A += p;
#pragma unroll
          for (int x = 0; x < D; ++x) acc[x] = fmaf(p, sm.vt[c][x], acc[x]);
        }
      }
    }
  };

  __shared__ bool mask[kTile];
  // stage 1: exact selected blocks, in chunks of kTile keys
  const int nsel = sm.nsel;
  for (int e = 0; e < nsel; ++e) {
    const int j = sm.list[e];
    const int ks0 = j * block, kc = block_count(j, L, block);
    for (int c0 = 0; c0 < kc; c0 += kTile) {
      const int ncols = min(kTile, kc - c0);
      __syncthreads();
      for (int idx = t; idx < ncols * D; idx += blockDim.x) {
        const size_t g = hoff + (size_t)(ks0 + c0) * D + idx;
        sm.kt[idx / D][idx % D] = to_f32(k[g]);
        sm.vt[idx / D][idx % D] = to_f32(v[g]);
      }
      for (int c = t; c < kTile; c += blockDim.x) mask[c] = c < ncols;
      __syncthreads();
      process_tile(ncols, false, mask);
    }
  }
  // stage 2: zeroth-order scan over the centroids of the unselected blocks
  const bool approx = (mode == PISA_MODE_PISA || mode == PISA_MODE_PER_BLOCK) && nsel < nb;
  if (approx) {
    const size_t so = (size_t)bh * nb * D;
    for (int j0 = 0; j0 < nb; j0 += kTile) {
      const int ncols = min(kTile, nb - j0);
      __syncthreads();
      for (int idx = t; idx < ncols * D; idx += blockDim.x) {
        sm.kt[idx / D][idx % D] = st.kbar[so + (size_t)j0 * D + idx];
        sm.vt[idx / D][idx % D] = st.vsum[so + (size_t)j0 * D + idx];
      }
      for (int c = t; c < kTile; c += blockDim.x) {
        const int j = j0 + c;
        mask[c] = c < ncols && !((sm.selbits[j >> 5] >> (j & 31)) & 1u);
        sm.w[c] = c < ncols ? (float)block_count(j, L, block) : 0.f;
      }
      __syncthreads();
      process_tile(ncols, true, mask);
    }
  }
  // stage 3 (per-block variant): N += s * alpha_tj * (q_t H_j) for every j in U_i, H_j streamed
  // through the key tile; m is final after stage 2, so alpha_tj = e^{s q_t.kbar_j - m}
  if (approx && mode == PISA_MODE_PER_BLOCK) {
    const size_t so = (size_t)bh * nb * D;
    for (int j = 0; j < nb; ++j) {
      if ((sm.selbits[j >> 5] >> (j & 31)) & 1u) continue;
      __syncthreads();
      for (int a = t; a < D; a += blockDim.x) sm.vt[0][a] = st.kbar[so + (size_t)j * D + a];
      __syncthreads();
      float f = 0.f;
      if (row_ok) {
        float dot = 0.f;
#pragma unroll 16
        for (int a = 0; a < D; ++a) dot = fmaf(sm.q[t][a], sm.vt[0][a], dot);
        f = scale * expf(scale * dot - m);
      }
      const float* hj = st.H + ((size_t)bh * nb + j) * D * D;
      for (int a0 = 0; a0 < D; a0 += kTile) {
        __syncthreads();
        for (int idx = t; idx < kTile * D; idx += blockDim.x) sm.kt[idx / D][idx % D] = hj[(size_t)a0 * D + idx];
        __syncthreads();
        if (row_ok) {
          for (int a = 0; a < kTile; ++a) {
            const float fa = f * sm.q[t][a0 + a];
#pragma unroll
            for (int c = 0; c < D; ++c) acc[c] = fmaf(fa, sm.kt[a][c], acc[c]);
          }
        }
      }
    }
  }
  // stage 3: first-order correction  N += s * A * (q_t Hbar), Hbar streamed through the key tile
  else if (approx) {
    const float* hb = st.hbar + (size_t)bh * D * D;
    for (int a0 = 0; a0 < D; a0 += kTile) {
      __syncthreads();
      for (int idx = t; idx < kTile * D; idx += blockDim.x) sm.kt[idx / D][idx % D] = hb[(size_t)a0 * D + idx];
      __syncthreads();
      if (row_ok) {
        for (int a = 0; a < kTile; ++a) {
          const float f = scale * A * sm.q[t][a0 + a];
#pragma unroll
          for (int c = 0; c < D; ++c) acc[c] = fmaf(f, sm.kt[a][c], acc[c]);
        }
      }
    }
  }
  if (row_ok) {
    const float inv = 1.f / l;
    T* orow = o + hoff + (size_t)(qs0 + t) * D;
#pragma unroll
    for (int c = 0; c < D; ++c) orow[c] = from_f32<T>(acc[c] * inv);
  }
}

template <typename T, int D>
cudaError_t run(const Dims& g, const void* q, const void* k, const void* v, const pisa_stats& st,
                const int32_t* sel, int keep_k, int mode, void* o, int* status, cudaStream_t stream) {
  const size_t smem = sizeof(Smem<D>);
  cudaError_t e;
  if ((e = set_max_dynamic_smem(reinterpret_cast<const void*>(attn_simt<T, D>), smem))) return e;
  attn_simt<T, D><<<dim3(g.nb, g.BH()), g.block, smem, stream>>>(
      static_cast<const T*>(q), static_cast<const T*>(k), static_cast<const T*>(v), st, sel, keep_k, mode, g.L,
      g.block, g.nb, g.scale, static_cast<T*>(o), status);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_attention_simt(const Dims& g, const void* q, const void* k, const void* v,
                                  const pisa_stats& st, const int32_t* sel, int keep_k, int mode, void* o,
                                  int* status, cudaStream_t stream) {
  if (g.dtype == PISA_FP32)
    return g.d == 64 ? run<float, 64>(g, q, k, v, st, sel, keep_k, mode, o, status, stream)
                     : run<float, 128>(g, q, k, v, st, sel, keep_k, mode, o, status, stream);
  return g.d == 64 ? run<__nv_bfloat16, 64>(g, q, k, v, st, sel, keep_k, mode, o, status, stream)
                   : run<__nv_bfloat16, 128>(g, q, k, v, st, sel, keep_k, mode, o, status, stream);
}

}  // namespace pisa
