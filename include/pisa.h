/*
 * pisa.h — C ABI of a B200 (sm_100a) library for piecewise sparse attention (PISA).
 *
 * Method: "PISA: Piecewise Sparse Attention Is Wiser for Efficient Diffusion Transformers"
 * (gist.science technical summary of arXiv 2602.01077), §2 방법론.  Key/value tokens of each
 * (batch, head) are cut into contiguous blocks of `block` tokens (the last may be shorter).  For
 * each query block i the router splits the key blocks into critical blocks S_i, attended exactly,
 * and the rest U_i, which still enter the same softmax numerator N_t and denominator D_t through
 *     alpha_{t,j} = exp(s q_t . kbar_j)                  (zeroth order, per block)
 *     N_t += sum_{j in U_i} alpha_{t,j} vsum_j + s (q_t Hbar) sum_{j in U_i} alpha_{t,j}
 *     D_t += sum_{j in U_i} cnt_j alpha_{t,j}
 * and o_t = N_t / D_t.  s is `softmax_scale`.
 *
 * Conventions shared by every entry point
 *   - q, k, v and o are dense row-major [B, H, L, d] tensors (d = head_dim for keys and values).
 *     They share one element type (`dtype`); o has the type of q.
 *   - Every pointer argument is a DEVICE pointer on the current CUDA device unless it is a
 *     `const pisa_shape*` / `pisa_stats*` (host structs) or documented otherwise.  The caller owns
 *     all memory; the library never allocates or frees device memory and keeps no pointer after a
 *     call returns.
 *   - Device pointers must be 16-byte aligned.  All work is enqueued on `stream` (0 = legacy
 *     default stream) and is asynchronous; the call returns once the kernels are enqueued.
 *   - Arguments are validated before anything is enqueued.  A call that returns an error status
 *     has enqueued nothing and written nothing.
 *   - No exceptions cross the ABI.  The library keeps no mutable host state apart from a cache of
 *     device attributes and resolved driver entry points.
 *   - Supported on the GPU: dtype PISA_BF16 or PISA_BF16_FP8QK with head_dim 128 and block 64 or
 *     128 (tensor-core path), and PISA_FP32 with head_dim 64 or 128 and block 64 or 128 (fp32 FMA
 *     path).
 */
#ifndef PISA_H_
#define PISA_H_

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define PISA_API __attribute__((visibility("default")))
#else
#define PISA_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

/* Same type as cudaStream_t / CUstream. */
typedef struct CUstream_st* pisa_stream_t;

typedef enum {
  PISA_OK = 0,
  PISA_ERR_INVALID_ARG = 1,    /* null/misaligned pointer, bad size, keep_k or lambda out of range */
  PISA_ERR_UNSUPPORTED = 2,    /* valid shape the GPU kernels do not implement (e.g. head_dim 96) */
  PISA_ERR_CUDA = 3,           /* a CUDA launch or driver call failed */
  PISA_ERR_DEVICE_TIMEOUT = 4  /* a kernel's bounded wait ran out (reported by pisa_read_device_error) */
} pisa_status;

/* PISA_BF16_FP8QK: q, k, v and o are bf16 as with PISA_BF16, but the attention logits (exact
 * and zeroth order) are computed on the tensor core from e4m3 copies that pisa_precompute writes:
 * q with one scale per row, k with one scale per key block, kbar with one scale per tile of 128
 * centroids; a group's scale is max|x| / 448 and x's code is e4m3(x / scale), both in float32.
 * Routing, the values and the first-order correction keep the bf16 / fp32 data.  A low-bit
 * exact stage in the spirit of PAROAttention's INT8/INT4 attention (its abstract); the pages
 * print no FP8 recipe.  head_dim 128 only; PISA_MODE_PER_BLOCK is not supported with it. */
typedef enum { PISA_BF16 = 0, PISA_FP32 = 1, PISA_BF16_FP8QK = 2 } pisa_dtype;

/* PISA_MODE_EXACT_ONLY drops U_i entirely (the keep-or-drop sparse attention the method is
 * compared against, §1 문제 정의); it needs keep_k >= 1.
 * PISA_MODE_PER_BLOCK replaces the global first-order term by each unselected block's own one,
 *     N_t += s sum_{j in U_i} alpha_{t,j} (q_t H_j)      instead of   s (q_t Hbar) sum_{j in U_i} alpha_{t,j},
 * the per-block form that §2 핵심 알고리즘 sets aside because it loads one d x d matrix per block.
 * It is a diagnostic of what the shared Hbar gives up; it needs the per-block matrices in the
 * stats (carved with with_H != 0 and written by pisa_precompute). */
typedef enum { PISA_MODE_PISA = 0, PISA_MODE_EXACT_ONLY = 1, PISA_MODE_PER_BLOCK = 2 } pisa_mode;

typedef struct {
  int32_t batch;          /* B >= 1 */
  int32_t heads;          /* H >= 1 */
  int32_t seq_len;        /* L >= 1 */
  int32_t head_dim;       /* d */
  int32_t block;          /* tokens per key block and per query block */
  int32_t dtype;          /* pisa_dtype of q, k, v, o */
  float   softmax_scale;  /* s > 0: multiplies every logit and the first-order correction */
} pisa_shape;

/* Per-head block statistics written by pisa_precompute.  nb = pisa_num_blocks(L, block).
 * All fp32 arrays are dense row-major.  The *_op arrays and vscale are tensor-core operand copies
 * and are used (and must be non-null) only when dtype == PISA_BF16: the softmax weights and the
 * values meet in an fp16 product (11 significant bits for the weights instead of bf16's 8), so the
 * values get an fp16 copy scaled by a per-head power of two that keeps every sum of a block in
 * range. */
typedef struct {
  float* qbar;     /* [B,H,nb,d]  mean of q over query block i                                */
  float* kbar;     /* [B,H,nb,d]  centroid of key block j                                      */
  float* vsum;     /* [B,H,nb,d]  sum of values of block j                                     */
  float* hbar;     /* [B,H,d,d]   Hbar[a][c]: mean over j of H_j, H_j = sum_n (k_n-kbar_j)^T v_n */
  float* M;        /* [B,H,nb]    ||H_j - Hbar||_F                                             */
  float* H;        /* nullable [B,H,nb,d,d]: per-block H_j, written only when non-null         */
  void*  kbar_op;  /* bf16 [B,H,nb,d]  kbar rounded to bf16                                    */
  void*  vsum_op;  /* fp16 [B,H,nb,d]  vsum / vscale, rounded to fp16                          */
  void*  hbar_op;  /* bf16 [B,H,d,d]   softmax_scale * Hbar^T, i.e. hbar_op[c][a]              */
  void*  v_op;     /* fp16 [B,H,L,d]   v / vscale (exact for every bf16 value in fp16 range)   */
  float* vscale;   /* [B,H]            power of two >= max|v| / 256 (1 when max|v| <= 256)     */
  void*  hdiff_op; /* nullable bf16 [B,H,nb,d,d]: softmax_scale * (H_j - Hbar), row a = key dim;
                    * written only when non-null (PISA_BF16 and with_H); PISA_MODE_PER_BLOCK reads it */
  /* PISA_BF16_FP8QK only (null otherwise): e4m3 codes (one byte each) and their float32 scales */
  void*  q8;       /* e4m3 [B,H,L,d]        q / qscale[row]                                      */
  void*  k8;       /* e4m3 [B,H,L,d]        k / kscale[block of the row]                         */
  void*  kbar8;    /* e4m3 [B,H,nb,d]       kbar / kbscale[j / 128]                              */
  float* qscale;   /* [B,H,L]               max_a |q_t,a| / 448 (1 for a zero row)               */
  float* kscale;   /* [B,H,nb]              max over block j of |k| / 448                        */
  float* kbscale;  /* [B,H,ceil(nb/128)]    max over the 128 centroids of a tile of |kbar| / 448 */
} pisa_stats;

/* ABI revision of this header. */
PISA_API int32_t pisa_abi_version(void);

/* nb = ceil(seq_len / block), or -1 if either argument is < 1. */
PISA_API int32_t pisa_num_blocks(int32_t seq_len, int32_t block);

/* Bytes of one contiguous buffer that pisa_stats_carve can split into every pisa_stats array
 * (H, and for PISA_BF16 hdiff_op, included when with_H != 0; the operand copies only for
 * PISA_BF16).  0 if the shape is invalid. */
PISA_API size_t pisa_stats_bytes(const pisa_shape* shape, int32_t with_H);

/* Host-only pointer arithmetic: fills *out with 256-byte-aligned sub-ranges of [base, base+bytes).
 * base must be 256-byte aligned; bytes >= pisa_stats_bytes(shape, with_H).  Enqueues nothing. */
PISA_API pisa_status pisa_stats_carve(const pisa_shape* shape, void* base, size_t bytes, int32_t with_H,
                             pisa_stats* out);

/* Device scratch bytes needed by pisa_precompute and pisa_attention for this shape (the first 256
 * bytes hold the device status word read by pisa_read_device_error; the rest is transient scratch:
 * partial sums in pisa_precompute, per-row softmax offsets in PISA_MODE_PER_BLOCK). */
PISA_API size_t pisa_workspace_bytes(const pisa_shape* shape);

/* Device scratch bytes that pisa_attention needs in PISA_MODE_PER_BLOCK (never less than
 * pisa_workspace_bytes): the status word, each row's softmax offset and 1/D_t, and the attention
 * output in fp32, B*H*L*d*4 bytes, so that o is rounded to bf16 only once.  0 if the shape is
 * invalid. */
PISA_API size_t pisa_perblock_workspace_bytes(const pisa_shape* shape);

/* Pre-computation (§2 하드웨어 구현, step 1; zeroth-order and global first-order bullets of
 * 핵심 알고리즘; M_j from 공분산 인식 라우팅): from q, k, v writes every array of *stats.
 * ws: device scratch of at least pisa_workspace_bytes(shape).  Its first 256 bytes hold the device
 * status word, which must be zero before the first call (allocate ws zeroed) and is cleared by
 * pisa_read_device_error; the rest need not be initialised.  Calls that share one ws must not run
 * concurrently.  Deterministic: fixed-order reductions, no floating-point atomics. */
PISA_API pisa_status pisa_precompute(const pisa_shape* shape, const void* q, const void* k, const void* v,
                            const pisa_stats* stats, void* ws, size_t ws_bytes, pisa_stream_t stream);

/* Zeroth-order pre-computation: the part of pisa_precompute that the zeroth-order Taylor term and
 * routing without the covariance term need (§2 핵심 알고리즘, zeroth-order bullet: block centroids
 * and value sums; the pooled queries of 공분산 인식 라우팅).  Writes qbar, kbar and vsum and, for
 * bf16 inputs, kbar_op, vsum_op, v_op and vscale (and the e4m3 copies for PISA_BF16_FP8QK); leaves
 * hbar, M, hbar_op, H and hdiff_op unwritten.  The statistics it writes equal pisa_precompute's bit
 * for bit.  What they serve: pisa_route with lambda == 0 (which does not read M) and pisa_attention
 * in PISA_MODE_EXACT_ONLY, i.e. a keep-or-drop pipeline, the baseline the method is measured
 * against (§1 문제 정의); PISA_MODE_PISA and PISA_MODE_PER_BLOCK need the full pisa_precompute.
 * It reads q, k and v once (no second pass over k and v, no first-order contractions).  Arguments,
 * ws and errors as for pisa_precompute. */
PISA_API pisa_status pisa_precompute_zeroth_order(const pisa_shape* shape, const void* q, const void* k,
                                                  const void* v, const pisa_stats* stats, void* ws,
                                                  size_t ws_bytes, pisa_stream_t stream);

/* pisa_precompute without a caller workspace, for callers that cannot allocate device memory (a
 * plugin whose host framework owns every device allocation, or a path that must not call cudaMalloc
 * because it may synchronise the device).  The method's description has no counterpart to this call;
 * it exists for such callers.  It runs the same kernels as pisa_precompute, with the scratch taken
 * from a fixed 16 MiB array in the library's device memory, which every device that loads the
 * library holds until the process exits.  It allocates nothing and frees nothing.
 *   - Arguments are checked first, exactly as by pisa_precompute (it takes no workspace, so there
 *     is no workspace check); then shapes whose pisa_workspace_bytes exceeds 16 MiB return
 *     PISA_ERR_UNSUPPORTED.  A rejected call enqueues nothing and does not touch the array.
 *   - The first call in a device's CUDA context looks up the array's device address there (a
 *     host-side CUDA runtime query); make that first call before any stream capture.  If the
 *     context is replaced (cudaDeviceReset), the next call looks the address up again.
 *   - Every call, on any stream, shares the one array: calls that overlap on the GPU race.  Each
 *     call clears the status word it uses before its kernels start; device-side wait timeouts of
 *     this call are not reported to the caller.
 * q, k, v, stats and stream as for pisa_precompute. */
PISA_API pisa_status pisa_precompute_noalloc(const pisa_shape* shape, const void* q, const void* k,
                                             const void* v, const pisa_stats* stats, pisa_stream_t stream);

/* Covariance-aware top-k routing (§2 공분산 인식 라우팅):
 *   s_ij = softmax_scale * qbar_i . kbar_j
 *   P_ij = cnt_j exp(s_ij) / sum_l cnt_l exp(s_il)
 *   r_ij = P_ij + lambda * M_j / sum_l M_l        (the M term is 0 when every M_j is 0)
 * sel    [B,H,nb,keep_k] int32: the keep_k largest r_ij of row i, ties to the lower j, ascending.
 * order  nullable [B,H,nb] int32: a permutation of the query blocks of each head that puts blocks
 *        with similar selections next to each other (pisa_attention runs consecutive pairs of it as
 *        one 128-row tile when block == 64; it changes no result).
 * scores nullable [B,H,nb,nb] fp32: r_ij.
 * Requires 0 <= keep_k <= nb, lambda finite and >= 0, nb <= 4096.  With lambda == 0 the M term is
 * dropped and stats->M is not read (it may be unwritten, as after pisa_precompute_zeroth_order). */
PISA_API pisa_status pisa_route(const pisa_shape* shape, const pisa_stats* stats, int32_t keep_k, float lambda,
                       int32_t* sel, int32_t* order, float* scores, pisa_stream_t stream);

/* pisa_precompute followed by pisa_route, with the same arguments, results and errors.
 * flags = 0: the separate calls.  flags = PISA_PRECOMPUTE_ROUTE_FUSED: for bf16 inputs (PISA_BF16,
 * PISA_BF16_FP8QK) with nb <= 128 (short sequences, where the fixed cost of pre-computation and
 * routing weighs most: §1 문제 정의, §4 실험 결과), one launch of a thread-block cluster per (batch,
 * head) whose CTAs meet at hardware cluster barriers between the passes (the e4m3 copies add their
 * quantization launch); every array it writes is bit-identical to what the separate calls write.
 * Otherwise, or when the device cannot make every head's cluster co-resident, it makes the
 * separate calls.  Measured on B200 the fused launch is not faster than the separate kernels
 * replayed as a CUDA graph (each pass is bound by its own per-CTA latency, not by launch gaps), so
 * it is not the default.  Any other flags value: PISA_ERR_INVALID_ARG.  ws as for pisa_precompute. */
#define PISA_PRECOMPUTE_ROUTE_FUSED 1
PISA_API pisa_status pisa_precompute_route(const pisa_shape* shape, const void* q, const void* k, const void* v,
                                           const pisa_stats* stats, int32_t keep_k, float lambda, int32_t* sel,
                                           int32_t* order, float* scores, void* ws, size_t ws_bytes,
                                           int32_t flags, pisa_stream_t stream);

/* Exact-or-approximate attention (§2: o_t = N_t / D_t and the numerator equation; 하드웨어 구현
 * stages 1-3: exact selected blocks, zeroth-order scan of the other blocks, global first-order
 * correction).  sel as written by pisa_route (ascending, distinct, < nb; checked on the device,
 * a bad entry sets the status word).  order: nullable, as written by pisa_route; null means
 * 0, 1, ..., nb-1.  o: [B,H,L,d] of dtype.  mode: pisa_mode.  ws as for pisa_precompute.
 * PISA_MODE_PER_BLOCK needs stats->hdiff_op (PISA_BF16) or stats->H (PISA_FP32) non-null and
 * written by the pisa_precompute call that wrote the other stats, and on the bf16 path ws_bytes >=
 * pisa_perblock_workspace_bytes(shape); otherwise PISA_ERR_INVALID_ARG.  On the bf16 path it is
 * two launches: the attention kernel, which leaves its fp32 output and each row's softmax offset
 * and 1/D_t in ws, then a tensor-core kernel that adds s sum_j alpha_{t,j} q_t (H_j - Hbar) / D_t
 * over the unselected blocks and writes o.  With keep_k == nb it is the PISA_MODE_PISA call. */
PISA_API pisa_status pisa_attention(const pisa_shape* shape, const void* q, const void* k, const void* v,
                           const pisa_stats* stats, const int32_t* sel, const int32_t* order,
                           int32_t keep_k, int32_t mode, void* o, void* ws, size_t ws_bytes,
                           pisa_stream_t stream);

/* Token reordering before blocking ("PAROAttention: Pattern-Aware ReOrdering for Efficient Sparse
 * and Quantized Attention in Visual Generation Models", abstract: reorder tokens so that attention
 * patterns become block-wise; the page gives no algorithm, and the reading built here permutes the
 * axis order of the video's frames x height x width grid, see pisa_axis_permutation).  Copies the
 * rows of src, a dense [batch_heads, seq_len, row_bytes] tensor, into dst:
 *   inverse == 0:  dst[h][i] = src[h][perm[i]]     (gather: reorder q, k, v before pisa_precompute)
 *   inverse != 0:  dst[h][perm[i]] = src[h][i]     (scatter: put the attention output back)
 * perm: device int32 [seq_len] shared by every head, or [batch_heads, seq_len] when
 * perm_per_head != 0; it must be a permutation of 0..seq_len-1 (an entry outside that range is
 * skipped and leaves its row of dst unwritten; a repeated entry leaves the result to write order).
 * row_bytes: a multiple of 16 (head_dim * element size).  src and dst must not overlap.  Byte copy:
 * any element type. */
PISA_API pisa_status pisa_permute_rows(const void* src, void* dst, const int32_t* perm, int32_t batch_heads,
                                       int32_t seq_len, int32_t row_bytes, int32_t perm_per_head, int32_t inverse,
                                       pisa_stream_t stream);

/* Host-only helper (perm_host is a HOST buffer of `capacity` int32, at least
 * frames*height*width + extra_tokens; a smaller capacity returns PISA_ERR_INVALID_ARG): the
 * permutation that lists the tokens of a frames x height x width grid, stored in raster order
 * (t slowest, then h, then w), in the axis order `order` — a NUL-terminated string of the three
 * distinct characters 't', 'h', 'w', slowest axis first ("thw" is the identity, "hwt" makes the
 * frame axis the fastest).  perm_host[i] = stored index of the token placed at position i.  The
 * extra_tokens rows after the grid (e.g. text tokens) keep their place at the end.  Enqueues
 * nothing; PISA_ERR_INVALID_ARG for a bad order or size. */
PISA_API pisa_status pisa_axis_permutation(int32_t frames, int32_t height, int32_t width, int32_t extra_tokens,
                                           const char* order, int32_t* perm_host, int64_t capacity);

/* Synchronises `stream`, copies the device status word out of ws into *code (0 = clean; otherwise
 * a PISA_DEVERR_* value below) and clears it.  Returns PISA_ERR_DEVICE_TIMEOUT when a bounded wait
 * ran out, PISA_ERR_INVALID_ARG for a bad selection entry, PISA_OK when clean. */
PISA_API pisa_status pisa_read_device_error(void* ws, int32_t* code, pisa_stream_t stream);

#define PISA_DEVERR_WAIT_TIMEOUT 1   /* an mbarrier wait exceeded its iteration limit */
#define PISA_DEVERR_BAD_SELECTION 2  /* sel held an entry out of range or out of order */

/* Static description of a status code. */
PISA_API const char* pisa_status_string(pisa_status status);

#ifdef __cplusplus
}
#endif

#endif /* PISA_H_ */
