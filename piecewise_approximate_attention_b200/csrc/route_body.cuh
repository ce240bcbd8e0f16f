// Internal: the bodies of the routing and pairing kernels (route.cu), shared with the fused
// short-sequence kernel (short_step_sm100.cu).
#pragma once

#include "common.cuh"

namespace pisa {
namespace {

constexpr int kRouteThreads = 256;
constexpr int kRouteWarps = kRouteThreads / 32;

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

// Scores of kRows query blocks against all nb centroids.  Each thread accumulates 8 query blocks x
// kCols centroids (jj, and jj + kRouteThreads / (kRows / 8) when kCols = 2); k̄ is streamed through
// shared memory in tiles of route_tile_j centroids x route_chunk columns (coalesced float4 loads,
// rows padded by 4 floats so that the float4 reads of 8 consecutive rows cover all 32 banks), the
// next chunk being loaded into registers while the current one is used.  Two centroids per thread
// halve the shared-memory reads per FMA but double the tile, which short rows of centroids (nb up
// to 256) would mostly leave empty.  Every score is summed over the columns in order, four at a
// time as fmaf(q.x, k.x, fmaf(q.y, k.y, fmaf(q.z, k.z, fmaf(q.w, k.w, acc)))).
template <int kRows>
constexpr int route_group_threads() { return kRouteThreads / (kRows / 8); }
template <int kRows, int kCols>
constexpr int route_tile_j() { return kCols * route_group_threads<kRows>(); }
template <int kRows>
constexpr int route_chunk() { return kRows == 16 ? 32 : 16; }
// centroids per thread for a head of nb key blocks
inline int route_cols(int nb) { return nb > 256 ? 2 : 1; }

// Body: routes query blocks [i0, i0 + rows) (rows <= kRows) of head bh with kRouteThreads threads;
// `smem` holds route_smem_floats<D, kRows>(nb) floats (16-byte aligned).  qbar, kbar and M are not
// __restrict__: the fused short-sequence kernel writes them earlier in the same launch, so they
// must be read through the coherent path.
template <int D, int kRows, int kCols>
__device__ __forceinline__ void route_rows(const float* qbar, const float* kbar, const float* M, int L, int block,
                                           int nb, float scale,
                                           int keep_k, float lam, int32_t* __restrict__ sel, float* __restrict__ scores,
                                           int bh, int i0, int rows, float* smem) {
  static_assert(kRows == 8 || kRows == 16, "8 query blocks per thread, one or two groups");
  static_assert(kCols == 1 || kCols == 2, "one or two centroids per thread");
  constexpr int kTPG = route_group_threads<kRows>();       // threads per group of 8 query blocks
  constexpr int kTileJ = route_tile_j<kRows, kCols>();
  constexpr int kChunk = route_chunk<kRows>();
  constexpr int kPitch = kChunk + 4;
  float* qs = smem;                                        // [kRows][D]
  float* ks = qs + kRows * D;                              // [kTileJ][kPitch]
  float* r = ks + kTileJ * kPitch;                         // [kRows][nb]
  uint32_t* hist = reinterpret_cast<uint32_t*>(r + kRows * nb);   // [kRouteWarps][256]: top-k histograms
  float* red = reinterpret_cast<float*>(hist + kRouteWarps * 256);     // [kRouteWarps]
  float* Ms = red + kRouteWarps;                                       // [nb]: M_j of this head
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const float* Mh = M ? M + (size_t)bh * nb : nullptr;    // null: lambda == 0, the M term is dropped

  static_assert(kRows * D % kRouteThreads == 0, "query rows per thread");
#pragma unroll
  for (int x = 0; x < kRows * D / kRouteThreads; ++x) {
    const int idx = threadIdx.x + x * kRouteThreads, ri = idx / D;
    qs[idx] = ri < rows ? scale * qbar[((size_t)bh * nb + i0 + ri) * D + idx % D] : 0.f;
  }
  // M_j kept in shared memory for the rows below; sum_l M_l in a fixed order
  float msum = 0.f;
#pragma unroll 4
  for (int j = threadIdx.x; j < nb; j += kRouteThreads) {
    const float mv = Mh ? Mh[j] : 0.f;
    Ms[j] = mv;
    msum += mv;
  }
  msum = warp_sum(msum);
  if (lane == 0) red[warp] = msum;

  const int jj = threadIdx.x % kTPG, g = threadIdx.x / kTPG;   // centroids jj (+ kTPG); query blocks 8g..8g+7
  const float4* kb4 = reinterpret_cast<const float4*>(kbar + (size_t)bh * nb * D);
  constexpr int kLoads = kTileJ * (kChunk / 4) / kRouteThreads;
  static_assert(kLoads * kRouteThreads == kTileJ * (kChunk / 4), "tile loads per thread");
  float4 nxt[kLoads];
  auto load_chunk = [&](int j0, int c0) {
#pragma unroll
    for (int x = 0; x < kLoads; ++x) {
      const int idx = threadIdx.x + x * kRouteThreads, jr = idx / (kChunk / 4), a4 = idx % (kChunk / 4);
      nxt[x] = j0 + jr < nb ? kb4[(size_t)(j0 + jr) * (D / 4) + c0 / 4 + a4] : make_float4(0.f, 0.f, 0.f, 0.f);
    }
  };
  load_chunk(0, 0);
  for (int j0 = 0; j0 < nb; j0 += kTileJ) {
    const int nj = min(kTileJ, nb - j0);
    // a warp whose centroids all lie past nb only helps with the loads
    const bool live = (jj - lane) < nj;
    float acc[8][kCols];
#pragma unroll
    for (int x = 0; x < 8; ++x)
#pragma unroll
      for (int c = 0; c < kCols; ++c) acc[x][c] = 0.f;
    for (int c0 = 0; c0 < D; c0 += kChunk) {
      __syncthreads();
#pragma unroll
      for (int x = 0; x < kLoads; ++x) {
        const int idx = threadIdx.x + x * kRouteThreads, jr = idx / (kChunk / 4), a4 = idx % (kChunk / 4);
        *reinterpret_cast<float4*>(ks + jr * kPitch + 4 * a4) = nxt[x];
      }
      __syncthreads();
      if (c0 + kChunk < D) load_chunk(j0, c0 + kChunk);
      else if (j0 + kTileJ < nb) load_chunk(j0 + kTileJ, 0);
      if (live) {
        const float* qg = qs + (8 * g) * D + c0;
#pragma unroll
        for (int a = 0; a < kChunk; a += 4) {
          float4 kv[kCols];
#pragma unroll
          for (int c = 0; c < kCols; ++c) kv[c] = *reinterpret_cast<const float4*>(ks + (jj + c * kTPG) * kPitch + a);
#pragma unroll
          for (int x = 0; x < 8; ++x) {
            const float4 qv = *reinterpret_cast<const float4*>(qg + x * D + a);
#pragma unroll
            for (int c = 0; c < kCols; ++c)
              acc[x][c] = fmaf(qv.x, kv[c].x, fmaf(qv.y, kv[c].y, fmaf(qv.z, kv[c].z, fmaf(qv.w, kv[c].w, acc[x][c]))));
          }
        }
      }
    }
#pragma unroll
    for (int c = 0; c < kCols; ++c) {
      const int jc = jj + c * kTPG;
      if (jc < nj) {
#pragma unroll
        for (int x = 0; x < 8; ++x) r[(8 * g + x) * nb + j0 + jc] = acc[x][c];
      }
    }
  }
  __syncthreads();
  msum = 0.f;
  for (int w = 0; w < kRouteWarps; ++w) msum += red[w];
  const float minv = msum > 0.f ? lam / msum : 0.f;

  const float last_cnt = (float)(L - (nb - 1) * block);
  for (int ri = warp; ri < rows; ri += kRouteWarps) {
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


template <int D, int kRows, int kCols>
constexpr size_t route_smem_floats(int nb) {
  return (size_t)kRows * D + (size_t)route_tile_j<kRows, kCols>() * (route_chunk<kRows>() + 4) + (size_t)kRows * nb +
         kRouteWarps * 256 + kRouteWarps + (size_t)nb;
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

// Body: pairs the query blocks of segment `seg` of head bh with kRouteThreads threads; `psm` holds
// pair_smem_bytes(nb) bytes.
__device__ __forceinline__ void pair_segment(const int32_t* __restrict__ sel, int nb, int keep_k,
                                             int32_t* __restrict__ order, int bh, int seg, uint32_t* psm) {
  const int nwords = (nb + 31) / 32;
  // word-major bitmaps: word w of block y at bits[w * kSeg + y], so a warp reading 32 consecutive
  // blocks' words touches 32 banks
  uint32_t* bits = psm;                                                  // [nwords][kSeg]
  uint16_t* ov = reinterpret_cast<uint16_t*>(bits + kSeg * nwords);     // [kSeg][kSeg], a < b used
  int32_t* singles = reinterpret_cast<int32_t*>(ov + kSeg * kSeg);      // [kSeg]
  __shared__ int npos_s, nsingle_s;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int s0 = seg * kSeg, n = min(kSeg, nb - s0);
  const int32_t* S = sel + ((size_t)bh * nb + s0) * keep_k;
  int32_t* out = order + (size_t)bh * nb + s0;
  for (int e = threadIdx.x; e < kSeg * nwords; e += kRouteThreads) bits[e] = 0u;
  __syncthreads();
  // the segment's selections are n * keep_k consecutive entries; sixteen loads per thread are in
  // flight before their atomics
  const int total = n * keep_k;
  for (int e0 = threadIdx.x; e0 < total; e0 += 16 * kRouteThreads) {
    int32_t jv[16];
#pragma unroll
    for (int x = 0; x < 16; ++x) jv[x] = e0 + x * kRouteThreads < total ? S[e0 + x * kRouteThreads] : -1;
#pragma unroll
    for (int x = 0; x < 16; ++x) {
      const int j = jv[x];
      if (j >= 0 && j < nb) atomicOr(&bits[(j >> 5) * kSeg + (e0 + x * kRouteThreads) / keep_k], 1u << (j & 31));
    }
  }
  __syncthreads();
  // overlaps |S_x ∩ S_y| for x < y < n (the only entries the pass below reads): a warp per row x,
  // its lanes over y
  for (int x = warp; x < n; x += kRouteWarps) {
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
  for (int e = threadIdx.x; e < nsingle_s; e += kRouteThreads) out[npos_s + e] = singles[e];
}

__host__ __device__ constexpr size_t pair_smem_bytes(int nb) {
  return (size_t)kSeg * ((nb + 31) / 32) * 4 + (size_t)kSeg * kSeg * 2 + (size_t)kSeg * 4;
}

}  // namespace
}  // namespace pisa
