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
#include "common.cuh"

namespace pisa {
namespace {

constexpr int kThreads = 256;
constexpr int kWarps = kThreads / 32;

__device__ __forceinline__ float warp_max(float x) {
  for (int o = 16; o > 0; o >>= 1) x = fmaxf(x, __shfl_xor_sync(0xffffffffu, x, o));
  return x;
}
__device__ __forceinline__ float warp_sum(float x) {
  for (int o = 16; o > 0; o >>= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
  return x;
}

// Selects the keep_k largest keys of u[0..nb) (ties to the lower index) and writes their indices,
// ascending, to out.  Runs on one warp; hist is a private 256-entry scratch.
__device__ void warp_topk(const uint32_t* u, int nb, int keep_k, uint32_t* hist, int32_t* out) {
  const int lane = threadIdx.x & 31;
  if (keep_k <= 0) return;
  uint32_t prefix = 0, pmask = 0;
  int want = keep_k;
  for (int shift = 24; shift >= 0; shift -= 8) {
    for (int b = lane; b < 256; b += 32) hist[b] = 0;
    __syncwarp();
    for (int j = lane; j < nb; j += 32)
      if ((u[j] & pmask) == prefix) atomicAdd(&hist[(u[j] >> shift) & 255u], 1u);
    __syncwarp();
    // lane l owns digits 255-8l .. 248-8l (descending); find the digit where the count of keys
    // with a larger-or-equal digit first reaches `want`.
    uint32_t cnt[8];
    uint32_t tot = 0;
#pragma unroll
    for (int t = 0; t < 8; ++t) { cnt[t] = hist[255 - 8 * lane - t]; tot += cnt[t]; }
    uint32_t incl = tot;
    for (int o = 1; o < 32; o <<= 1) {
      uint32_t y = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += y;
    }
    const uint32_t excl = incl - tot;
    int found_digit = -1;
    uint32_t above = 0;
    if (excl < (uint32_t)want && incl >= (uint32_t)want) {
      uint32_t run = excl;
#pragma unroll
      for (int t = 0; t < 8; ++t) {
        if (found_digit < 0 && run + cnt[t] >= (uint32_t)want) { found_digit = 255 - 8 * lane - t; above = run; }
        run += cnt[t];
      }
    }
    const unsigned owner = __ballot_sync(0xffffffffu, found_digit >= 0);
    const int src = __ffs(owner) - 1;
    found_digit = __shfl_sync(0xffffffffu, found_digit, src);
    above = __shfl_sync(0xffffffffu, above, src);
    want -= (int)above;
    prefix |= (uint32_t)found_digit << shift;
    pmask |= 255u << shift;
    __syncwarp();
  }
  // prefix is now the exact key of the keep_k-th largest element; `want` of its equals are taken.
  const unsigned lt = (1u << lane) - 1u;
  int pos = 0, eq_seen = 0;
  for (int j0 = 0; j0 < nb; j0 += 32) {
    const int j = j0 + lane;
    const uint32_t key = j < nb ? u[j] : 0u;
    const bool gt = j < nb && key > prefix;
    const bool eq = j < nb && key == prefix;
    const unsigned eqm = __ballot_sync(0xffffffffu, eq);
    const bool take = gt || (eq && eq_seen + __popc(eqm & lt) < want);
    const unsigned tm = __ballot_sync(0xffffffffu, take);
    if (take) out[pos + __popc(tm & lt)] = j;
    pos += __popc(tm);
    eq_seen += __popc(eqm);
  }
}

// Scores of kRows query blocks against all nb centroids: k̄ is streamed through shared memory in
// tiles of kTileJ = 4 * kThreads / kRows rows (coalesced float4 loads, rows padded by 4 floats so
// the float4 reads of 32 different rows are conflict-free); each thread accumulates 4 query blocks
// x 1 centroid.
template <int kRows>
constexpr int tile_j() { return 4 * kThreads / kRows; }

template <int D, int kRows>
__global__ void __launch_bounds__(kThreads, 2) route_kernel(const float* __restrict__ qbar, const float* __restrict__ kbar,
                                                         const float* __restrict__ M, int L, int block, int nb,
                                                         float scale, int keep_k, float lam,
                                                         int32_t* __restrict__ sel, float* __restrict__ scores) {
  constexpr int kTileJ = tile_j<kRows>();
  extern __shared__ __align__(16) float smem[];
  float* qs = smem;                                        // [kRows][D]
  float* ks = qs + kRows * D;                              // [kTileJ][D + 4]
  float* r = ks + kTileJ * (D + 4);                        // [kRows][nb]
  uint32_t* hist = reinterpret_cast<uint32_t*>(r + kRows * nb);   // [kWarps][256]
  float* red = reinterpret_cast<float*>(hist + kWarps * 256);     // [kWarps]
  float* Ms = red + kWarps;                                       // [nb]: M_j of this head
  const int bh = blockIdx.y, i0 = blockIdx.x * kRows;
  const int rows = min(kRows, nb - i0);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const float* Mh = M ? M + (size_t)bh * nb : nullptr;    // null: lambda == 0, the M term is dropped

  static_assert(kRows * D % kThreads == 0, "query rows per thread");
#pragma unroll
  for (int x = 0; x < kRows * D / kThreads; ++x) {
    const int idx = threadIdx.x + x * kThreads, ri = idx / D;
    qs[idx] = ri < rows ? scale * qbar[((size_t)bh * nb + i0 + ri) * D + idx % D] : 0.f;
  }
  // M_j kept in shared memory for the rows below; sum_l M_l in a fixed order
  float msum = 0.f;
#pragma unroll 4
  for (int j = threadIdx.x; j < nb; j += kThreads) {
    const float mv = Mh ? Mh[j] : 0.f;
    Ms[j] = mv;
    msum += mv;
  }
  msum = warp_sum(msum);
  if (lane == 0) red[warp] = msum;

  const int jj = threadIdx.x % kTileJ, g = threadIdx.x / kTileJ;   // centroid column, query group
  const float4* kb4 = reinterpret_cast<const float4*>(kbar + (size_t)bh * nb * D);
  // the next k̄ tile is loaded into registers while the current one is used
  constexpr int kLoads = kTileJ * (D / 4) / kThreads;
  static_assert(kLoads * kThreads == kTileJ * (D / 4), "tile loads per thread");
  float4 nxt[kLoads];
  auto load_tile = [&](int j0) {
#pragma unroll
    for (int x = 0; x < kLoads; ++x) {
      const int idx = threadIdx.x + x * kThreads, jr = idx / (D / 4), a4 = idx % (D / 4);
      nxt[x] = j0 + jr < nb ? kb4[(size_t)(j0 + jr) * (D / 4) + a4] : make_float4(0.f, 0.f, 0.f, 0.f);
    }
  };
  load_tile(0);
  for (int j0 = 0; j0 < nb; j0 += kTileJ) {
    const int nj = min(kTileJ, nb - j0);
    __syncthreads();
#pragma unroll
    for (int x = 0; x < kLoads; ++x) {
      const int idx = threadIdx.x + x * kThreads, jr = idx / (D / 4), a4 = idx % (D / 4);
      *reinterpret_cast<float4*>(ks + jr * (D + 4) + 4 * a4) = nxt[x];
    }
    __syncthreads();
    if (j0 + kTileJ < nb) load_tile(j0 + kTileJ);
    float acc[4] = {0.f, 0.f, 0.f, 0.f};
    const float* kr = ks + jj * (D + 4);
#pragma unroll 8
    for (int a = 0; a < D; a += 4) {
      const float4 kv = *reinterpret_cast<const float4*>(kr + a);
#pragma unroll
      for (int x = 0; x < 4; ++x) {
        const float4 qv = *reinterpret_cast<const float4*>(qs + (4 * g + x) * D + a);
        acc[x] = fmaf(qv.x, kv.x, fmaf(qv.y, kv.y, fmaf(qv.z, kv.z, fmaf(qv.w, kv.w, acc[x]))));
      }
    }
    if (jj < nj) {
#pragma unroll
      for (int x = 0; x < 4; ++x) r[(4 * g + x) * nb + j0 + jj] = acc[x];
    }
  }
  __syncthreads();
  msum = 0.f;
  for (int w = 0; w < kWarps; ++w) msum += red[w];
  const float minv = msum > 0.f ? lam / msum : 0.f;

  const float last_cnt = (float)(L - (nb - 1) * block);
  for (int ri = warp; ri < rows; ri += kWarps) {
    float* rr = r + ri * nb;
    float mx = -INFINITY;
    for (int j = lane; j < nb; j += 32) mx = fmaxf(mx, rr[j]);
    mx = warp_max(mx);
    float den = 0.f;
    for (int j = lane; j < nb; j += 32) {
      const float w = (j == nb - 1 ? last_cnt : (float)block) * expf(rr[j] - mx);
      rr[j] = w;
      den += w;
    }
    den = warp_sum(den);
    const float inv = 1.f / den;
    const size_t row = (size_t)bh * nb + i0 + ri;
    for (int j = lane; j < nb; j += 32) {
      const float val = rr[j] * inv + minv * Ms[j];
      rr[j] = val;
      if (scores) scores[row * nb + j] = val;
    }
    __syncwarp();
    warp_topk(reinterpret_cast<const uint32_t*>(rr), nb, keep_k, hist + warp * 256, sel + row * keep_k);
  }
}

// Query-block pairing for 128-row tiles when block == 64.  The query blocks are cut into segments
// of kSeg consecutive blocks, one CTA each; inside a segment a greedy pass in index order pairs each
// unpaired block i with the unpaired block p of the same segment (p > i) whose selection shares the
// most key blocks with S_i (ties to the nearer p).  Pairs fill the segment's range of the order
// first, blocks left without a partner follow, so no tile straddles two segments (a full segment
// holds an even count).  The attention result does not depend on the order; only the union of S_i
// and S_p, which one tile iterates over, does.  Bitmaps of the selections live in shared memory.
constexpr int kSeg = 128;
static_assert(kSeg == 128, "the pairing pass keeps a segment's set of paired blocks in four 32-bit words");

// Bit b of a 128-bit set held as four words in registers (the same value in every lane).
__device__ __forceinline__ bool bit128(uint32_t u0, uint32_t u1, uint32_t u2, uint32_t u3, int b) {
  const int w = b >> 5;
  const uint32_t x = w == 0 ? u0 : (w == 1 ? u1 : (w == 2 ? u2 : u3));
  return (x >> (b & 31)) & 1u;
}

__global__ void __launch_bounds__(kThreads) pair_kernel(const int32_t* __restrict__ sel, int nb, int keep_k,
                                                        int32_t* __restrict__ order) {
  extern __shared__ uint32_t psm[];
  const int nwords = (nb + 31) / 32;
  // word-major bitmaps: word w of block y at bits[w * kSeg + y], so a warp reading 32 consecutive
  // blocks' words touches 32 banks
  uint32_t* bits = psm;                                                  // [nwords][kSeg]
  uint16_t* ov = reinterpret_cast<uint16_t*>(bits + kSeg * nwords);     // [kSeg][kSeg], a < b used
  int32_t* singles = reinterpret_cast<int32_t*>(ov + kSeg * kSeg);      // [kSeg]
  __shared__ int npos_s, nsingle_s;
  const int bh = blockIdx.y, lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int s0 = blockIdx.x * kSeg, n = min(kSeg, nb - s0);
  const int32_t* S = sel + ((size_t)bh * nb + s0) * keep_k;
  int32_t* out = order + (size_t)bh * nb + s0;
  for (int e = threadIdx.x; e < kSeg * nwords; e += kThreads) bits[e] = 0u;
  __syncthreads();
  // the segment's selections are n * keep_k consecutive entries; sixteen loads per thread are in
  // flight before their atomics
  const int total = n * keep_k;
  for (int e0 = threadIdx.x; e0 < total; e0 += 16 * kThreads) {
    int32_t jv[16];
#pragma unroll
    for (int x = 0; x < 16; ++x) jv[x] = e0 + x * kThreads < total ? S[e0 + x * kThreads] : -1;
#pragma unroll
    for (int x = 0; x < 16; ++x) {
      const int j = jv[x];
      if (j >= 0 && j < nb) atomicOr(&bits[(j >> 5) * kSeg + (e0 + x * kThreads) / keep_k], 1u << (j & 31));
    }
  }
  __syncthreads();
  // overlaps |S_x ∩ S_y| for x < y < n (the only entries the pass below reads): a warp per row x,
  // its lanes over y
  for (int x = warp; x < n; x += kWarps) {
    for (int y = x + 1 + lane; y < n; y += 32) {
      int cnt = 0;
      for (int w = 0; w < nwords; ++w) cnt += __popc(bits[w * kSeg + x] & bits[w * kSeg + y]);
      ov[x * kSeg + y] = (uint16_t)cnt;
    }
  }
  __syncthreads();
  if (warp == 0) {
    // The set of paired blocks and the output counts stay in registers: u0..u3 identical in every
    // lane (for the test on a), and each lane's own view of its four blocks lane + 32 x (bit x of
    // `avail` set while that block is unpaired), so a candidate test is one bit of one register.
    uint32_t u0 = 0u, u1 = 0u, u2 = 0u, u3 = 0u;
    uint32_t avail = 0u;
#pragma unroll
    for (int x = 0; x < kSeg / 32; ++x) avail |= lane + 32 * x < n ? 1u << x : 0u;
    int npos = 0, nsingle = 0;
    for (int a = 0; a < n; ++a) {
      if (bit128(u0, u1, u2, u3, a)) continue;
      // best partner packed as ((overlap + 1) << 8) | (255 - distance): one warp max picks it (0 = none)
      const uint16_t* row = ov + a * kSeg;
      uint32_t key = 0u;
#pragma unroll
      for (int x = 0; x < kSeg / 32; ++x) {
        const int b = lane + 32 * x;
        if (b > a && ((avail >> x) & 1u)) key = max(key, ((row[b] + 1u) << 8) | (uint32_t)(255 - (b - a)));
      }
      key = __reduce_max_sync(0xffffffffu, key);
      const int pb = key ? a + 255 - (int)(key & 255u) : a;
      if (lane == (a & 31)) avail &= ~(1u << (a >> 5));
      if (lane == (pb & 31)) avail &= ~(1u << (pb >> 5));
#pragma unroll
      for (int m = 0; m < 2; ++m) {
        const int x = m ? pb : a;
        const uint32_t bit = 1u << (x & 31);
        const int w = x >> 5;
        u0 |= w == 0 ? bit : 0u;
        u1 |= w == 1 ? bit : 0u;
        u2 |= w == 2 ? bit : 0u;
        u3 |= w == 3 ? bit : 0u;
      }
      if (key) {
        if (lane == 0) {
          out[npos] = s0 + a;
          out[npos + 1] = s0 + pb;
        }
        npos += 2;
      } else {
        if (lane == 0) singles[nsingle] = s0 + a;
        ++nsingle;
      }
    }
    if (lane == 0) {
      npos_s = npos;
      nsingle_s = nsingle;
    }
  }
  __syncthreads();
  for (int e = threadIdx.x; e < nsingle_s; e += kThreads) out[npos_s + e] = singles[e];
}

__global__ void identity_order(int nb, int32_t* __restrict__ order) {
  const int bh = blockIdx.y;
  for (int i = blockIdx.x * blockDim.x + threadIdx.x; i < nb; i += gridDim.x * blockDim.x)
    order[(size_t)bh * nb + i] = i;
}

template <int D, int kRows>
cudaError_t launch_route_kernel(const Dims& g, const pisa_stats& st, int keep_k, float lam, int32_t* sel,
                                float* scores, cudaStream_t stream) {
  const size_t smem = ((size_t)kRows * D + (size_t)tile_j<kRows>() * (D + 4) + (size_t)kRows * g.nb) * sizeof(float) +
                      kWarps * 256 * sizeof(uint32_t) + kWarps * sizeof(float) + (size_t)g.nb * sizeof(float);
  cudaError_t e;
  if ((e = cudaFuncSetAttribute(route_kernel<D, kRows>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem)))
    return e;
  // lambda == 0 drops the M term: M is not read (it may be unwritten)
  route_kernel<D, kRows><<<dim3((g.nb + kRows - 1) / kRows, g.BH()), kThreads, smem, stream>>>(
      st.qbar, st.kbar, lam > 0.f ? st.M : nullptr, g.L, g.block, g.nb, g.scale, keep_k, lam, sel, scores);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_route(const Dims& g, const pisa_stats& st, int keep_k, float lam, int32_t* sel,
                         int32_t* order, float* scores, cudaStream_t stream) {
  cudaError_t e;
  // 16 query blocks per CTA while their score rows fit comfortably in shared memory, else 8
  if (g.d == 64)
    e = g.nb <= 2048 ? launch_route_kernel<64, 16>(g, st, keep_k, lam, sel, scores, stream)
                     : launch_route_kernel<64, 8>(g, st, keep_k, lam, sel, scores, stream);
  else
    e = g.nb <= 2048 ? launch_route_kernel<128, 16>(g, st, keep_k, lam, sel, scores, stream)
                     : launch_route_kernel<128, 8>(g, st, keep_k, lam, sel, scores, stream);
  if (e != cudaSuccess) return e;
  if (order) {
    if (g.block == 64 && keep_k > 0 && g.nb > 2) {
      const int nwords = (g.nb + 31) / 32;
      const size_t psmem = (size_t)kSeg * nwords * 4 + (size_t)kSeg * kSeg * 2 + (size_t)kSeg * 4;
      if ((e = cudaFuncSetAttribute(pair_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)psmem))) return e;
      pair_kernel<<<dim3((g.nb + kSeg - 1) / kSeg, g.BH()), kThreads, psmem, stream>>>(sel, g.nb, keep_k, order);
    } else {
      identity_order<<<dim3((g.nb + 255) / 256, g.BH()), 256, 0, stream>>>(g.nb, order);
    }
    if ((e = cudaGetLastError())) return e;
  }
  return cudaSuccess;
}

}  // namespace pisa
