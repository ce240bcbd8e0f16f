// Block statistics with fp32 FMA arithmetic: qbar, kbar, vsum, H_j, Hbar, M_j.
//
// "PISA: Piecewise Sparse Attention Is Wiser for Efficient Diffusion Transformers", §2 방법론:
// the pre-computation step of the fused pipeline (하드웨어 구현 step 1) produces the block
// centroids kbar_j and value sums used by the zeroth-order term, and the global statistic Hbar,
// the average over all blocks of the block-wise first-order matrices H_j = sum_n (k_n-kbar_j)^T v_n,
// used by the first-order correction.  Covariance-aware routing (공분산 인식 라우팅) also needs
// M_j = ||H_j - Hbar|| (Frobenius).
//
// Three launches, all deterministic (fixed-order sums, no atomics):
//   1. stats_partial: one CTA per (head, group of kBlocksPerPart key blocks) writes the per-block
//      means/sums and the group's partial sum of H_j.
//   2. hbar_reduce:   sums the partials of each head in order, divides by nb.
//   3. cov_norm:      one CTA per (head, key block) recomputes H_j and reduces ||H_j - Hbar||_F^2.
// This path serves fp32 inputs; bf16 inputs use the tensor-core kernels.
#include "common.cuh"

namespace pisa {
namespace {

constexpr int kThreads = 256;

// Loads rows [s, s+cnt) of one head into shared memory as fp32 (row stride D).
template <typename T, int D>
__device__ void load_rows(const T* __restrict__ src, int s, int cnt, float* dst) {
  for (int idx = threadIdx.x; idx < cnt * D; idx += kThreads) dst[idx] = to_f32(src[(size_t)s * D + idx]);
}

// acc[r] += sum_n Kc[n][a_r] * V[n][c] with a_r = tid / D + r * (kThreads / D), c = tid % D.
template <int D>
__device__ __forceinline__ void accumulate_H(const float* Kc, const float* Vs, int cnt, float* acc) {
  constexpr int kStep = kThreads / D;
  constexpr int R = D * D / kThreads;
  const int a0 = threadIdx.x / D, c = threadIdx.x % D;
  for (int n = 0; n < cnt; ++n) {
    const float vc = Vs[n * D + c];
#pragma unroll
    for (int r = 0; r < R; ++r) acc[r] = fmaf(Kc[n * D + a0 + r * kStep], vc, acc[r]);
  }
}

// Block means/sums of block j; leaves the centred keys in Ks and kbar in kb.
template <typename T, int D>
__device__ void block_moments(const T* q, const T* k, const T* v, int j, int L, int block,
                              float* Ks, float* Vs, float* kb, float* qb, float* vb) {
  const int s = j * block, cnt = block_count(j, L, block);
  load_rows<T, D>(k, s, cnt, Ks);
  load_rows<T, D>(v, s, cnt, Vs);
  __syncthreads();
  const int c = threadIdx.x;
  if (c < D) {
    float sk = 0.f, sv = 0.f;
    for (int n = 0; n < cnt; ++n) { sk += Ks[n * D + c]; sv += Vs[n * D + c]; }
    kb[c] = sk / (float)cnt;
    vb[c] = sv;
  } else if (c - D < D && qb) {
    const int cc = c - D;
    float sq = 0.f;
    for (int n = 0; n < cnt; ++n) sq += to_f32(q[(size_t)(s + n) * D + cc]);
    qb[cc] = sq / (float)cnt;
  }
  __syncthreads();
  for (int idx = threadIdx.x; idx < cnt * D; idx += kThreads) Ks[idx] -= kb[idx % D];
  __syncthreads();
}

// kFirstOrder = false: the zeroth-order statistics only (no partial sums of H_j).
template <typename T, int D, bool kFirstOrder>
__global__ void __launch_bounds__(kThreads) stats_partial(const T* __restrict__ q, const T* __restrict__ k,
                                                          const T* __restrict__ v, int L, int block, int nb,
                                                          pisa_stats st, float* __restrict__ partials) {
  extern __shared__ float smem[];
  float* Ks = smem;                 // [block][D]
  float* Vs = Ks + block * D;       // [block][D]
  float* kb = Vs + block * D;       // [D]
  float* qb = kb + D;               // [D]
  float* vb = qb + D;               // [D]
  constexpr int R = D * D / kThreads;
  const int part = blockIdx.x, bh = blockIdx.y, nparts = gridDim.x;
  const size_t hoff = (size_t)bh * L * D;
  float acc[R];
#pragma unroll
  for (int r = 0; r < R; ++r) acc[r] = 0.f;
  const int j0 = part * kBlocksPerPart, j1 = min(nb, j0 + kBlocksPerPart);
  for (int j = j0; j < j1; ++j) {
    block_moments<T, D>(q + hoff, k + hoff, v + hoff, j, L, block, Ks, Vs, kb, qb, vb);
    const size_t so = ((size_t)bh * nb + j) * D;
    for (int c = threadIdx.x; c < D; c += kThreads) {
      st.kbar[so + c] = kb[c];
      st.vsum[so + c] = vb[c];
      st.qbar[so + c] = qb[c];
    }
    if (kFirstOrder) accumulate_H<D>(Ks, Vs, block_count(j, L, block), acc);
    __syncthreads();
  }
  if (!kFirstOrder) return;
  constexpr int kStep = kThreads / D;
  const int a0 = threadIdx.x / D, c = threadIdx.x % D;
  float* out = partials + ((size_t)bh * nparts + part) * D * D;
#pragma unroll
  for (int r = 0; r < R; ++r) out[(a0 + r * kStep) * D + c] = acc[r];
}

// Per head: Hbar = (sum of the group partials of H_j, in order) / nb, its bf16 operand copy, and
// (when vmax is given) the value scale: the smallest power of two >= max|v| / 256, so that
// v / vscale and every block sum of it (at most 128 terms) fit comfortably in fp16.
// One thread per four consecutive elements; the partials are read eight at a time (all loads in
// flight together) and added in group order, so the sum is the same as a plain loop's.
// Launched with programmatic stream serialization after the pass that writes the partials, it
// lets the next kernel start at once and waits for the partials before it reads them.
template <int D>
__global__ void __launch_bounds__(kThreads) hbar_reduce(const float* __restrict__ partials, int nparts, int nb,
                                                        float scale, float* __restrict__ hbar,
                                                        __nv_bfloat16* __restrict__ hbar_op,
                                                        const float* __restrict__ vmax, float* __restrict__ vscale) {
  constexpr int kVec = D * D / 4;
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  asm volatile("griddepcontrol.wait;" ::: "memory");
  const int e4 = blockIdx.x * kThreads + threadIdx.x, bh = blockIdx.y;
  if (vmax && vscale && blockIdx.x == 0 && threadIdx.x == 0) {
    float mx = 0.f;
    for (int i = 0; i < nparts; ++i) mx = fmaxf(mx, vmax[(size_t)bh * nparts + i]);
    float sc = 1.f;
    while (mx > 256.f * sc && sc < 0x1p100f) sc *= 2.f;
    vscale[bh] = sc;
  }
  if (e4 >= kVec) return;
  const float4* p = reinterpret_cast<const float4*>(partials + (size_t)bh * nparts * D * D) + e4;
  float4 s = make_float4(0.f, 0.f, 0.f, 0.f);
  for (int i = 0; i < nparts; i += 8) {
    float4 x[8];
#pragma unroll
    for (int u = 0; u < 8; ++u)
      if (i + u < nparts) x[u] = __ldcg(p + (size_t)(i + u) * kVec);
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      if (i + u < nparts) {
        s.x += x[u].x;
        s.y += x[u].y;
        s.z += x[u].z;
        s.w += x[u].w;
      }
    }
  }
  const float fnb = (float)nb;
  const float4 h = make_float4(s.x / fnb, s.y / fnb, s.z / fnb, s.w / fnb);
  reinterpret_cast<float4*>(hbar + (size_t)bh * D * D)[e4] = h;
  if (hbar_op) {
    const int a = (4 * e4) / D, c = (4 * e4) % D;
    __nv_bfloat16* op = hbar_op + (size_t)bh * D * D + a;
    op[(size_t)(c + 0) * D] = __float2bfloat16_rn(scale * h.x);
    op[(size_t)(c + 1) * D] = __float2bfloat16_rn(scale * h.y);
    op[(size_t)(c + 2) * D] = __float2bfloat16_rn(scale * h.z);
    op[(size_t)(c + 3) * D] = __float2bfloat16_rn(scale * h.w);
  }
}

template <typename T, int D>
__global__ void __launch_bounds__(kThreads) cov_norm(const T* __restrict__ k, const T* __restrict__ v, int L,
                                                     int block, int nb, pisa_stats st) {
  extern __shared__ float smem[];
  float* Ks = smem;
  float* Vs = Ks + block * D;
  float* kb = Vs + block * D;
  float* red = kb + 3 * D;          // [kThreads / 32]
  constexpr int R = D * D / kThreads;
  constexpr int kStep = kThreads / D;
  const int j = blockIdx.x, bh = blockIdx.y;
  const size_t hoff = (size_t)bh * L * D;
  block_moments<T, D>(nullptr, k + hoff, v + hoff, j, L, block, Ks, Vs, kb, nullptr, kb + D);
  float acc[R];
#pragma unroll
  for (int r = 0; r < R; ++r) acc[r] = 0.f;
  accumulate_H<D>(Ks, Vs, block_count(j, L, block), acc);
  const int a0 = threadIdx.x / D, c = threadIdx.x % D;
  const float* hb = st.hbar + (size_t)bh * D * D;
  float* Hout = st.H ? st.H + ((size_t)bh * nb + j) * D * D : nullptr;
  float ss = 0.f;
#pragma unroll
  for (int r = 0; r < R; ++r) {
    const int e = (a0 + r * kStep) * D + c;
    const float dlt = acc[r] - hb[e];
    ss = fmaf(dlt, dlt, ss);
    if (Hout) Hout[e] = acc[r];
  }
  for (int o = 16; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = ss;
  __syncthreads();
  if (threadIdx.x == 0) {
    float t = 0.f;
    for (int w = 0; w < kThreads / 32; ++w) t += red[w];
    st.M[(size_t)bh * nb + j] = sqrtf(t);
  }
}

template <typename T, int D>
cudaError_t run(const Dims& g, const void* q, const void* k, const void* v, const pisa_stats& st, void* ws,
                bool first_order, cudaStream_t stream) {
  const int nparts = num_parts(g);
  float* partials = reinterpret_cast<float*>(static_cast<char*>(ws) + kStatusBytes);
  const size_t smem_a = ((size_t)2 * g.block * D + 3 * D) * sizeof(float);
  const size_t smem_c = ((size_t)2 * g.block * D + 3 * D + kThreads / 32) * sizeof(float);
  cudaError_t e;
  if ((e = set_max_dynamic_smem(reinterpret_cast<const void*>(stats_partial<T, D, true>), smem_a)))
    return e;
  if ((e = set_max_dynamic_smem(reinterpret_cast<const void*>(stats_partial<T, D, false>), smem_a)))
    return e;
  if ((e = set_max_dynamic_smem(reinterpret_cast<const void*>(cov_norm<T, D>), smem_c)))
    return e;
  if (!first_order) {
    stats_partial<T, D, false><<<dim3(nparts, g.BH()), kThreads, smem_a, stream>>>(
        static_cast<const T*>(q), static_cast<const T*>(k), static_cast<const T*>(v), g.L, g.block, g.nb, st, partials);
    return cudaGetLastError();
  }
  stats_partial<T, D, true><<<dim3(nparts, g.BH()), kThreads, smem_a, stream>>>(
      static_cast<const T*>(q), static_cast<const T*>(k), static_cast<const T*>(v), g.L, g.block, g.nb, st, partials);
  hbar_reduce<D><<<dim3((D * D / 4 + kThreads - 1) / kThreads, g.BH()), kThreads, 0, stream>>>(
      partials, nparts, g.nb, g.scale, st.hbar, static_cast<__nv_bfloat16*>(st.hbar_op), nullptr, nullptr);
  cov_norm<T, D><<<dim3(g.nb, g.BH()), kThreads, smem_c, stream>>>(
      static_cast<const T*>(k), static_cast<const T*>(v), g.L, g.block, g.nb, st);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_hbar_reduce(const Dims& g, const float* partials, int nparts, const float* vmax,
                               const pisa_stats& st, cudaStream_t stream, bool pdl) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((g.d * g.d / 4 + kThreads - 1) / kThreads, g.BH());
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = 0;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = pdl ? 1 : 0;
  __nv_bfloat16* hop = static_cast<__nv_bfloat16*>(st.hbar_op);
  if (g.d == 64)
    return cudaLaunchKernelEx(&cfg, hbar_reduce<64>, partials, nparts, g.nb, g.scale, st.hbar, hop, vmax, st.vscale);
  return cudaLaunchKernelEx(&cfg, hbar_reduce<128>, partials, nparts, g.nb, g.scale, st.hbar, hop, vmax, st.vscale);
}

cudaError_t launch_precompute_simt(const Dims& g, const void* q, const void* k, const void* v,
                                   const pisa_stats& st, void* ws, bool first_order, cudaStream_t stream) {
  if (g.dtype == PISA_FP32) {
    return g.d == 64 ? run<float, 64>(g, q, k, v, st, ws, first_order, stream)
                     : run<float, 128>(g, q, k, v, st, ws, first_order, stream);
  }
  return g.d == 64 ? run<__nv_bfloat16, 64>(g, q, k, v, st, ws, first_order, stream)
                   : run<__nv_bfloat16, 128>(g, q, k, v, st, ws, first_order, stream);
}

}  // namespace pisa
