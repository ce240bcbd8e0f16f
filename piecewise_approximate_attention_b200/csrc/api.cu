// Host entry points of the C ABI declared in pisa.h: validation, buffer carving, dispatch.
#include <cmath>
#include <cstring>

#include "common.cuh"
#include "pisa_testing.h"

namespace pisa {
namespace {

constexpr int kMaxBlocks = 4096;

// test-only fault injection (pisa_testing.h)
int g_test_fault = PISA_TESTING_FAULT_NONE;
unsigned long long g_test_wait_ns = 0;
int g_test_pre_fault = PISA_TESTING_FAULT_NONE;
unsigned long long g_test_pre_wait_ns = 0;

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// Validates the shape; fills g.  Returns INVALID_ARG for impossible shapes and UNSUPPORTED for
// shapes the GPU kernels do not implement.
pisa_status check_shape(const pisa_shape* s, Dims* g) {
  if (!s) return PISA_ERR_INVALID_ARG;
  if (s->batch < 1 || s->heads < 1 || s->seq_len < 1 || s->head_dim < 1 || s->block < 1)
    return PISA_ERR_INVALID_ARG;
  if (s->dtype != PISA_BF16 && s->dtype != PISA_FP32 && s->dtype != PISA_BF16_FP8QK) return PISA_ERR_INVALID_ARG;
  if (!std::isfinite(s->softmax_scale) || !(s->softmax_scale > 0.f)) return PISA_ERR_INVALID_ARG;
  if (s->head_dim != 64 && s->head_dim != 128) return PISA_ERR_UNSUPPORTED;
  if (bf16_inputs(s->dtype) && s->head_dim != 128) return PISA_ERR_UNSUPPORTED;
  if (s->block != 64 && s->block != 128) return PISA_ERR_UNSUPPORTED;
  const long long nb = ((long long)s->seq_len + s->block - 1) / s->block;
  if (nb > kMaxBlocks) return PISA_ERR_UNSUPPORTED;
  if ((long long)s->batch * s->heads > 65535) return PISA_ERR_UNSUPPORTED;
  g->B = s->batch;
  g->H = s->heads;
  g->L = s->seq_len;
  g->d = s->head_dim;
  g->block = s->block;
  g->nb = (int)nb;
  g->dtype = s->dtype;
  g->scale = s->softmax_scale;
  return PISA_OK;
}

pisa_status check_stats(const Dims& g, const pisa_stats* st, bool need_ops) {
  if (!st) return PISA_ERR_INVALID_ARG;
  const void* req[] = {st->qbar, st->kbar, st->vsum, st->hbar, st->M};
  for (const void* p : req)
    if (!p || !aligned16(p)) return PISA_ERR_INVALID_ARG;
  if ((st->H && !aligned16(st->H)) || (st->hdiff_op && !aligned16(st->hdiff_op))) return PISA_ERR_INVALID_ARG;
  if (need_ops && bf16_inputs(g.dtype)) {
    const void* ops[] = {st->kbar_op, st->vsum_op, st->hbar_op, st->v_op, st->vscale};
    for (const void* p : ops)
      if (!p || !aligned16(p)) return PISA_ERR_INVALID_ARG;
  }
  if (need_ops && g.dtype == PISA_BF16_FP8QK) {
    const void* f8[] = {st->q8, st->k8, st->kbar8, st->qscale, st->kscale, st->kbscale};
    for (const void* p : f8)
      if (!p || !aligned16(p)) return PISA_ERR_INVALID_ARG;
  }
  return PISA_OK;
}

pisa_status cuda_status(cudaError_t e) { return e == cudaSuccess ? PISA_OK : PISA_ERR_CUDA; }

size_t round_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

constexpr int kStatsArrays = 18;

// Sizes of the stats arrays in carve order.
void stats_sizes(const Dims& g, int with_H, size_t out[kStatsArrays]) {
  const size_t bh = (size_t)g.BH(), nb = (size_t)g.nb, d = (size_t)g.d;
  const bool ops = bf16_inputs(g.dtype);
  const bool f8 = g.dtype == PISA_BF16_FP8QK;
  out[0] = bh * nb * d * 4;            // qbar
  out[1] = bh * nb * d * 4;            // kbar
  out[2] = bh * nb * d * 4;            // vsum
  out[3] = bh * d * d * 4;             // hbar
  out[4] = bh * nb * 4;                // M
  out[5] = with_H ? bh * nb * d * d * 4 : 0;  // H
  out[6] = ops ? bh * nb * d * 2 : 0;  // kbar_op
  out[7] = ops ? bh * nb * d * 2 : 0;  // vsum_op
  out[8] = ops ? bh * d * d * 2 : 0;   // hbar_op
  out[9] = ops ? bh * (size_t)g.L * d * 2 : 0;   // v_op
  out[10] = ops ? bh * 4 : 0;          // vscale
  out[11] = (ops && with_H) ? bh * nb * d * d * 2 : 0;   // hdiff_op
  out[12] = f8 ? bh * (size_t)g.L * d : 0;               // q8
  out[13] = f8 ? bh * (size_t)g.L * d : 0;               // k8
  out[14] = f8 ? bh * nb * d : 0;                        // kbar8
  out[15] = f8 ? bh * (size_t)g.L * 4 : 0;               // qscale
  out[16] = f8 ? bh * nb * 4 : 0;                        // kscale
  out[17] = f8 ? bh * ((nb + 127) / 128) * 4 : 0;        // kbscale
}

}  // namespace

pisa_status validate_precompute(const pisa_shape* shape, const void* q, const void* k, const void* v,
                                const pisa_stats* stats, Dims* g) {
  pisa_status s = check_shape(shape, g);
  if (s != PISA_OK) return s;
  if (!q || !k || !v || !aligned16(q) || !aligned16(k) || !aligned16(v)) return PISA_ERR_INVALID_ARG;
  return check_stats(*g, stats, true);
}

}  // namespace pisa

using namespace pisa;

extern "C" {

int32_t pisa_abi_version(void) { return 7; }

int32_t pisa_num_blocks(int32_t seq_len, int32_t block) {
  if (seq_len < 1 || block < 1) return -1;
  return (int32_t)(((long long)seq_len + block - 1) / block);
}

size_t pisa_stats_bytes(const pisa_shape* shape, int32_t with_H) {
  Dims g;
  if (check_shape(shape, &g) != PISA_OK) return 0;
  size_t sz[kStatsArrays];
  stats_sizes(g, with_H, sz);
  size_t tot = 0;
  for (size_t s : sz) tot += round_up(s, 256);
  return tot;
}

pisa_status pisa_stats_carve(const pisa_shape* shape, void* base, size_t bytes, int32_t with_H, pisa_stats* out) {
  Dims g;
  pisa_status s = check_shape(shape, &g);
  if (s != PISA_OK) return s;
  if (!base || !out || (reinterpret_cast<uintptr_t>(base) & 255u)) return PISA_ERR_INVALID_ARG;
  if (bytes < pisa_stats_bytes(shape, with_H)) return PISA_ERR_INVALID_ARG;
  size_t sz[kStatsArrays];
  stats_sizes(g, with_H, sz);
  char* p = static_cast<char*>(base);
  void* ptr[kStatsArrays];
  for (int i = 0; i < kStatsArrays; ++i) {
    ptr[i] = sz[i] ? p : nullptr;
    p += round_up(sz[i], 256);
  }
  pisa_stats st;
  st.qbar = static_cast<float*>(ptr[0]);
  st.kbar = static_cast<float*>(ptr[1]);
  st.vsum = static_cast<float*>(ptr[2]);
  st.hbar = static_cast<float*>(ptr[3]);
  st.M = static_cast<float*>(ptr[4]);
  st.H = static_cast<float*>(ptr[5]);
  st.kbar_op = ptr[6];
  st.vsum_op = ptr[7];
  st.hbar_op = ptr[8];
  st.v_op = ptr[9];
  st.vscale = static_cast<float*>(ptr[10]);
  st.hdiff_op = ptr[11];
  st.q8 = ptr[12];
  st.k8 = ptr[13];
  st.kbar8 = ptr[14];
  st.qscale = static_cast<float*>(ptr[15]);
  st.kscale = static_cast<float*>(ptr[16]);
  st.kbscale = static_cast<float*>(ptr[17]);
  *out = st;
  return PISA_OK;
}

size_t pisa_workspace_bytes(const pisa_shape* shape) {
  Dims g;
  if (check_shape(shape, &g) != PISA_OK) return 0;
  const size_t pre = round_up(partials_bytes(g), 256) + round_up(vmax_bytes(g), 256);
  const size_t rows = round_up(rowstats_bytes(g), 256);
  return kStatusBytes + (pre > rows ? pre : rows);
}

size_t pisa_perblock_workspace_bytes(const pisa_shape* shape) {
  Dims g;
  if (check_shape(shape, &g) != PISA_OK) return 0;
  const size_t base = pisa_workspace_bytes(shape);
  const size_t pb = perblock_ws_bytes(g);
  return pb > base ? pb : base;
}

namespace {
pisa_status precompute(const pisa_shape* shape, const void* q, const void* k, const void* v, const pisa_stats* stats,
                       void* ws, size_t ws_bytes, bool first_order, pisa_stream_t stream) {
  Dims g;
  pisa_status s = validate_precompute(shape, q, k, v, stats, &g);
  if (s != PISA_OK) return s;
  if (!ws || !aligned16(ws) || ws_bytes < pisa_workspace_bytes(shape)) return PISA_ERR_INVALID_ARG;
  cudaStream_t cs = reinterpret_cast<cudaStream_t>(stream);
  if (bf16_inputs(g.dtype)) {
    cudaError_t e = launch_precompute_sm100(g, q, k, v, *stats, ws, first_order,
                                            g_test_pre_wait_ns ? g_test_pre_wait_ns : kWaitLimitNs, g_test_pre_fault, cs);
    if (e == cudaSuccess && g.dtype == PISA_BF16_FP8QK) e = launch_quantize_fp8(g, q, k, *stats, cs);
    return cuda_status(e);
  }
  return cuda_status(launch_precompute_simt(g, q, k, v, *stats, ws, first_order, cs));
}
}  // namespace

pisa_status pisa_precompute(const pisa_shape* shape, const void* q, const void* k, const void* v,
                            const pisa_stats* stats, void* ws, size_t ws_bytes, pisa_stream_t stream) {
  return precompute(shape, q, k, v, stats, ws, ws_bytes, true, stream);
}

pisa_status pisa_precompute_zeroth_order(const pisa_shape* shape, const void* q, const void* k, const void* v,
                                         const pisa_stats* stats, void* ws, size_t ws_bytes, pisa_stream_t stream) {
  return precompute(shape, q, k, v, stats, ws, ws_bytes, false, stream);
}

namespace {
pisa_status check_route_args(const Dims& g, int32_t keep_k, float lambda, const int32_t* sel, const int32_t* order,
                             const float* scores) {
  if (keep_k < 0 || keep_k > g.nb || !std::isfinite(lambda) || lambda < 0.f) return PISA_ERR_INVALID_ARG;
  if ((keep_k > 0 && (!sel || !aligned16(sel))) || (order && !aligned16(order)) || (scores && !aligned16(scores)))
    return PISA_ERR_INVALID_ARG;
  return PISA_OK;
}
}  // namespace

pisa_status pisa_route(const pisa_shape* shape, const pisa_stats* stats, int32_t keep_k, float lambda,
                       int32_t* sel, int32_t* order, float* scores, pisa_stream_t stream) {
  Dims g;
  pisa_status s = check_shape(shape, &g);
  if (s != PISA_OK) return s;
  if ((s = check_stats(g, stats, false)) != PISA_OK) return s;
  if ((s = check_route_args(g, keep_k, lambda, sel, order, scores)) != PISA_OK) return s;
  return cuda_status(launch_route(g, *stats, keep_k, lambda, sel, order, scores,
                                  reinterpret_cast<cudaStream_t>(stream)));
}

pisa_status pisa_precompute_route(const pisa_shape* shape, const void* q, const void* k, const void* v,
                                  const pisa_stats* stats, int32_t keep_k, float lambda, int32_t* sel,
                                  int32_t* order, float* scores, void* ws, size_t ws_bytes, int32_t flags,
                                  pisa_stream_t stream) {
  Dims g;
  pisa_status s = validate_precompute(shape, q, k, v, stats, &g);
  if (s != PISA_OK) return s;
  if (!ws || !aligned16(ws) || ws_bytes < pisa_workspace_bytes(shape)) return PISA_ERR_INVALID_ARG;
  if ((s = check_route_args(g, keep_k, lambda, sel, order, scores)) != PISA_OK) return s;
  if (flags != 0 && flags != PISA_PRECOMPUTE_ROUTE_FUSED) return PISA_ERR_INVALID_ARG;
  cudaStream_t cs = reinterpret_cast<cudaStream_t>(stream);
  bool launched = false;
  cudaError_t e = cudaSuccess;
  if (flags == PISA_PRECOMPUTE_ROUTE_FUSED)
    e = launch_short_step_sm100(g, q, k, v, *stats, ws, keep_k, lambda, sel, order, scores, cs, &launched);
  if (e != cudaSuccess) return PISA_ERR_CUDA;
  if (launched) {
    if (g.dtype == PISA_BF16_FP8QK) e = launch_quantize_fp8(g, q, k, *stats, cs);
    return cuda_status(e);
  }
  if ((s = pisa_precompute(shape, q, k, v, stats, ws, ws_bytes, stream)) != PISA_OK) return s;
  return pisa_route(shape, stats, keep_k, lambda, sel, order, scores, stream);
}

pisa_status pisa_attention(const pisa_shape* shape, const void* q, const void* k, const void* v,
                           const pisa_stats* stats, const int32_t* sel, const int32_t* order, int32_t keep_k,
                           int32_t mode, void* o, void* ws, size_t ws_bytes, pisa_stream_t stream) {
  Dims g;
  pisa_status s = check_shape(shape, &g);
  if (s != PISA_OK) return s;
  if (!q || !k || !v || !o || !ws || !aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) ||
      !aligned16(ws))
    return PISA_ERR_INVALID_ARG;
  if (mode != PISA_MODE_PISA && mode != PISA_MODE_EXACT_ONLY && mode != PISA_MODE_PER_BLOCK)
    return PISA_ERR_INVALID_ARG;
  if (keep_k < 0 || keep_k > g.nb || (mode == PISA_MODE_EXACT_ONLY && keep_k < 1)) return PISA_ERR_INVALID_ARG;
  if (keep_k > 0 && (!sel || !aligned16(sel))) return PISA_ERR_INVALID_ARG;
  if (order && !aligned16(order)) return PISA_ERR_INVALID_ARG;
  if ((s = check_stats(g, stats, true)) != PISA_OK) return s;
  if (mode == PISA_MODE_PER_BLOCK && g.dtype == PISA_BF16_FP8QK) return PISA_ERR_UNSUPPORTED;
  if (mode == PISA_MODE_PER_BLOCK && !(g.dtype == PISA_BF16 ? stats->hdiff_op : stats->H)) return PISA_ERR_INVALID_ARG;
  if (ws_bytes < pisa_workspace_bytes(shape)) return PISA_ERR_INVALID_ARG;
  const bool per_block = mode == PISA_MODE_PER_BLOCK && keep_k < g.nb;
  if (per_block && g.dtype == PISA_BF16 && ws_bytes < pisa_perblock_workspace_bytes(shape)) return PISA_ERR_INVALID_ARG;
  int* status = static_cast<int*>(ws);
  cudaStream_t cs = reinterpret_cast<cudaStream_t>(stream);
  if (bf16_inputs(g.dtype)) {
    AttnMaps maps;
    const uint64_t bh = (uint64_t)g.BH();
    if (!encode_bf16_3d(&maps.q, q, g.d, g.L, bh, g.block) || !encode_bf16_3d(&maps.k, k, g.d, g.L, bh, g.block) ||
        !encode_16bit_3d(&maps.v, stats->v_op, g.d, g.L, bh, g.block, true) ||
        !encode_bf16_3d(&maps.kbar, stats->kbar_op, g.d, g.nb, bh, 128) ||
        !encode_16bit_3d(&maps.vsum, stats->vsum_op, g.d, g.nb, bh, 128, true) ||
        !encode_bf16_3d(&maps.hbar, stats->hbar_op, g.d, g.d, bh, 128))
      return PISA_ERR_CUDA;
    F8Scales f8;
    if (g.dtype == PISA_BF16_FP8QK) {
      if (!encode_u8_3d(&maps.q8, stats->q8, g.d, g.L, bh, g.block) ||
          !encode_u8_3d(&maps.k8, stats->k8, g.d, g.L, bh, g.block) ||
          !encode_u8_3d(&maps.kbar8, stats->kbar8, g.d, g.nb, bh, 128))
        return PISA_ERR_CUDA;
      f8.q = stats->qscale;
      f8.k = stats->kscale;
      f8.kb = stats->kbscale;
    }
    const unsigned long long wait_ns = g_test_wait_ns ? g_test_wait_ns : kWaitLimitNs;
    // per-block mode: the attention kernel runs in PISA mode, leaves each row's softmax offset and
    // 1/D_t and its fp32 output in ws; the second kernel adds the per-block minus global first-order
    // difference and writes o (one rounding to bf16)
    char* wsb = static_cast<char*>(ws);
    float2* rows = per_block ? reinterpret_cast<float2*>(wsb + kStatusBytes) : nullptr;
    float* o32 = per_block ? reinterpret_cast<float*>(wsb + o32_offset(g)) : nullptr;
    cudaError_t e = launch_attention_sm100(g, maps, sel, order, keep_k, mode == PISA_MODE_EXACT_ONLY ? mode : PISA_MODE_PISA,
                                           stats->vscale, f8, o, rows, o32, status, wait_ns, g_test_fault, cs);
    if (e != cudaSuccess || !per_block) return cuda_status(e);
    CUtensorMap hmap;
    if (!encode_bf16_3d(&hmap, stats->hdiff_op, g.d, (uint64_t)g.nb * g.d, bh, 128)) return PISA_ERR_CUDA;
    return cuda_status(launch_perblock_sm100(g, maps, hmap, sel, order, keep_k, rows, o32, o, status, wait_ns, cs));
  }
  return cuda_status(launch_attention_simt(g, q, k, v, *stats, sel, keep_k, mode, o, status, cs));
}

pisa_status pisa_permute_rows(const void* src, void* dst, const int32_t* perm, int32_t batch_heads, int32_t seq_len,
                              int32_t row_bytes, int32_t perm_per_head, int32_t inverse, pisa_stream_t stream) {
  if (!src || !dst || !perm || !aligned16(src) || !aligned16(dst) || !aligned16(perm)) return PISA_ERR_INVALID_ARG;
  if (batch_heads < 1 || batch_heads > 65535 || seq_len < 1 || row_bytes < 16 || row_bytes % 16) return PISA_ERR_INVALID_ARG;
  const uintptr_t a = reinterpret_cast<uintptr_t>(src), b = reinterpret_cast<uintptr_t>(dst);
  const uintptr_t n = (uintptr_t)batch_heads * (uintptr_t)seq_len * (uintptr_t)row_bytes;
  if (a < b + n && b < a + n) return PISA_ERR_INVALID_ARG;   // overlapping buffers
  return cuda_status(launch_permute_rows(src, dst, perm, batch_heads, seq_len, row_bytes, perm_per_head ? 1 : 0,
                                         inverse ? 1 : 0, reinterpret_cast<cudaStream_t>(stream)));
}

pisa_status pisa_axis_permutation(int32_t frames, int32_t height, int32_t width, int32_t extra_tokens,
                                  const char* order, int32_t* perm_host, int64_t capacity) {
  if (frames < 1 || height < 1 || width < 1 || extra_tokens < 0 || !order || !perm_host) return PISA_ERR_INVALID_ARG;
  const long long total = (long long)frames * height * width + extra_tokens;
  if (total > 0x7fffffffLL || capacity < total) return PISA_ERR_INVALID_ARG;
  // order: the three axes t, h, w, slowest first
  int axis[3], seen = 0;
  for (int i = 0; i < 3; ++i) {
    const char c = order[i];
    const int ax = c == 't' ? 0 : c == 'h' ? 1 : c == 'w' ? 2 : -1;
    if (ax < 0 || (seen >> ax) & 1) return PISA_ERR_INVALID_ARG;
    seen |= 1 << ax;
    axis[i] = ax;
  }
  if (order[3] != '\0') return PISA_ERR_INVALID_ARG;
  const int ext[3] = {frames, height, width};
  // raster (t, h, w) strides of the stored sequence
  const long long stride[3] = {(long long)height * width, width, 1};
  const int n0 = ext[axis[0]], n1 = ext[axis[1]], n2 = ext[axis[2]];
  long long pos = 0;
  for (int i0 = 0; i0 < n0; ++i0)
    for (int i1 = 0; i1 < n1; ++i1)
      for (int i2 = 0; i2 < n2; ++i2)
        perm_host[pos++] = (int32_t)(i0 * stride[axis[0]] + i1 * stride[axis[1]] + i2 * stride[axis[2]]);
  for (int e = 0; e < extra_tokens; ++e, ++pos) perm_host[pos] = (int32_t)pos;
  return PISA_OK;
}

pisa_status pisa_read_device_error(void* ws, int32_t* code, pisa_stream_t stream) {
  if (!ws || !code || !aligned16(ws)) return PISA_ERR_INVALID_ARG;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  int32_t host = 0;
  if (cudaMemcpyAsync(&host, ws, sizeof(int32_t), cudaMemcpyDeviceToHost, st) != cudaSuccess) return PISA_ERR_CUDA;
  if (cudaMemsetAsync(ws, 0, sizeof(int32_t), st) != cudaSuccess) return PISA_ERR_CUDA;
  if (cudaStreamSynchronize(st) != cudaSuccess) return PISA_ERR_CUDA;
  *code = host;
  if (host == 0) return PISA_OK;
  return host == PISA_DEVERR_WAIT_TIMEOUT ? PISA_ERR_DEVICE_TIMEOUT : PISA_ERR_INVALID_ARG;
}

pisa_status pisa_testing_set_attention_fault(int32_t fault, uint64_t wait_limit_ns) {
  if (fault != PISA_TESTING_FAULT_NONE && fault != PISA_TESTING_FAULT_SKIP_Q_LOAD) return PISA_ERR_INVALID_ARG;
  g_test_fault = fault;
  g_test_wait_ns = wait_limit_ns;
  return PISA_OK;
}

pisa_status pisa_testing_set_precompute_fault(int32_t fault, uint64_t wait_limit_ns) {
  if (fault != PISA_TESTING_FAULT_NONE && fault != PISA_TESTING_FAULT_SKIP_TILE_LOAD) return PISA_ERR_INVALID_ARG;
  g_test_pre_fault = fault;
  g_test_pre_wait_ns = wait_limit_ns;
  return PISA_OK;
}

const char* pisa_status_string(pisa_status status) {
  switch (status) {
    case PISA_OK: return "ok";
    case PISA_ERR_INVALID_ARG: return "invalid argument";
    case PISA_ERR_UNSUPPORTED: return "unsupported shape or dtype";
    case PISA_ERR_CUDA: return "CUDA error";
    case PISA_ERR_DEVICE_TIMEOUT: return "device-side bounded wait timed out";
  }
  return "unknown status";
}

}  // extern "C"
