/*
 * q8.h -- C ABI of libq8: Q8_0 single-token decode and the fused MoE
 * up/gate + SwiGLU feed-forward step, as hand-written CUDA for B200 (sm_100a).
 *
 * The operations follow two web pages:
 *  [HADA]  "GPUなしで13年前のXeon上でGemma 4 26Bを毎秒5トークンで実行する"
 *          (news.hada.io), sections 「非AVX2ビルドで壊れていた演算パス」
 *          (the MOE_FUSED_UP_GATE / FUSED_UP_GATE ops), 「3段階で構成された修正」
 *          (combined up_gate_exps [n_embd, 2*n_ff, n_experts], first half gate,
 *          second half up; view_3d slices; mul_mat_id per slice;
 *          fused_mul_unary(gate, up, SILU); quantize_row_q8_0_x4) and
 *          「原因を絞り込んだ過程」 (ggml_vec_dot_q8_0_q8_0).
 *  [NARR]  "narray-llm" README, section "Llama 2 110M を int8 (Q8_0) で"
 *          (Q8_0 single-token decode).
 *
 * Q8_0 (layout not printed on the pages; the reading used throughout): blocks
 * of 32 int8 values q along the contiguous axis with one fp16 scale d; a value
 * is d * q.  Quantization of a block: amax = max|x|, d32 = amax / 127 (fp32),
 * q = round-half-away-from-zero(x * (1 / d32)) (q = 0 when d32 == 0), stored
 * d = fp16 round-to-nearest-even of d32.  The block dot is the exact int32
 * sum of q_w * q_x; a row result is sum_b d_w,b * d_x,b * isum_b.
 *
 * Conventions for every call:
 *  - Every pointer is a DEVICE pointer unless its comment says host.  The
 *    caller allocates and owns every buffer; the library allocates nothing,
 *    frees nothing and keeps no device memory between calls.
 *  - Calls are asynchronous on `stream` (a cudaStream_t passed as void*; NULL
 *    is the legacy default stream) and return after enqueueing.  Except
 *    q8_check, no call synchronizes or copies to the host.
 *  - Arguments are validated on the host before anything is launched.  A
 *    non-Q8_OK return means nothing was launched and no output was touched.
 *  - Errors found on the device (bad routing ids) are latched in the caller's
 *    workspace and reported by q8_check.
 *  - A shape without a kernel returns Q8_E_UNSUPPORTED: there is no fallback
 *    to another device or to the CPU, and no partial dispatch.
 *  - Results are deterministic: the same inputs give bitwise-equal outputs
 *    (no floating-point atomics; every sum has a fixed order).
 *  - Accuracy: block dots are exact int32; every fp32 output of a matmul lies
 *    within 1e-5 * sum|w * x| (the sum of the dequantized products' magnitudes)
 *    of the exact value of its definition.  Which kernel runs depends on the
 *    shape: experts with >= 4 routed rows in a call, and dense calls with
 *    16..32 activation rows, run on the int8 tensor cores
 *    (tcgen05.mma.kind::i8) when 128 <= k <= 4096 (and, for up/gate, n_ff is
 *    a multiple of 64, and no g_out/u_out is asked for); the rest run on
 *    the dp4a streaming kernels.  The two round their fp32 sums differently, so the same row can
 *    differ in its last bits between a call where its expert crosses the
 *    16-row line and one where it does not; both are within the bound.
 *  - Thread safety: calls may come from several host threads on different
 *    streams; the library holds no mutable global state except a per-thread
 *    detail string for the last error.
 */
#ifndef Q8_H
#define Q8_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Status codes. */
typedef enum {
    Q8_OK = 0,
    Q8_E_NULL = 1,        /* a required pointer is NULL                                  */
    Q8_E_SHAPE = 2,       /* k % 32 != 0, a size < 1 or above its limit, shapes disagree */
    Q8_E_ALIGN = 3,       /* a pointer or stride breaks its alignment rule               */
    Q8_E_BAD_ID = 4,      /* (device) a routing id outside [0, n_mat) or repeated in a token */
    Q8_E_UNSUPPORTED = 5, /* a valid request that no kernel here implements             */
    Q8_E_CUDA = 6,        /* a CUDA runtime call or launch failed                         */
    Q8_E_WORKSPACE = 7    /* workspace NULL or smaller than the *_workspace_size answer   */
} q8_status;

/* Limits checked by the host validation. */
#define Q8_QK 32                /* weights per block                                   */
#define Q8_MAX_K 16384          /* longest row (elements)                               */
#define Q8_MAX_USED 32          /* routed experts per token                             */
#define Q8_MAX_GEMV_DESC 128    /* problems in one q8_gemv_batched call                 */

/*
 * A packed Q8_0 weight tensor in device memory (a non-owning view).
 *  qs: int8 quants; element (m, r, i) at qs[(m * mat_stride + r) * k + i].
 *      Rows are k bytes apart; qs must be 16-byte aligned.
 *  d:  fp16 scale bits; scale (m, r, b) at d[(m * mat_stride + r) * ld_d + b],
 *      b < k/32.  ld_d >= k/32 and ld_d % 8 == 0 (every scale row starts on a
 *      16-byte boundary); d must be 16-byte aligned.
 *  k:  row length in elements, a multiple of 32, <= Q8_MAX_K.
 *  rows: rows of each matrix (output features).
 *  n_mat: number of matrices (experts); 1 for a dense weight.
 *  mat_stride: rows from one matrix to the next, >= rows.  A tensor packed by
 *      q8_pack has mat_stride == rows.  The gate half of a combined up_gate
 *      tensor (rows 0..n_ff-1 of each expert) is the view {qs, d, k, n_ff,
 *      n_exp, ld_d, 2*n_ff}; the up half is the same view with qs and d
 *      advanced by n_ff rows ([HADA] 「3段階で構成された修正」: view_3d slices).
 */
typedef struct {
    const int8_t *qs;
    const uint16_t *d;
    int64_t k;
    int64_t rows;
    int64_t n_mat;
    int64_t ld_d;
    int64_t mat_stride;
} q8_tensor;

/* Scale-row stride (in fp16 elements) that q8_pack writes for row length k:
 * k/32 rounded up to a multiple of 8.  Returns 0 if k is not a positive
 * multiple of 32. */
int64_t q8_scale_stride(int64_t k);

/*
 * q8_pack -- quantize an fp32 weight matrix to packed Q8_0 (setup step).
 *  w:   fp32 [n_rows][k] row-major (for a 3-D ggml tensor [k, rows, n_mat],
 *       n_rows = rows * n_mat with the matrix index outermost); 16-byte aligned.
 *  qs:  out int8 [n_rows][k]; d: out fp16 bits [n_rows][ld_d], the entries
 *       b >= k/32 of each row written as 0.  Both 16-byte aligned.
 *  ld_d: >= k/32, multiple of 8 (use q8_scale_stride(k)).
 * Same quantization rule as q8_quantize_row.
 */
q8_status q8_pack(const float *w, int64_t n_rows, int64_t k, int8_t *qs, uint16_t *d,
                  int64_t ld_d, void *stream);

/*
 * q8_pack_up_gate -- pack separate gate and up weights into the combined
 * up/gate layout (setup step).  [HADA] 「3段階で構成された修正」: when the gate
 * and up weights are already separate tensors, the step is silu(W_gate x) *
 * (W_up x); here they are packed once into the combined tensor, and the one
 * fused up/gate kernel serves both forms.
 *  w_gate, w_up: fp32 [n_mat][n_ff][k] each (n_mat == 1 for a dense layer);
 *       16-byte aligned.
 *  qs:  out int8 [n_mat][2*n_ff][k]: in each matrix, rows 0..n_ff-1 are the
 *       gate rows and rows n_ff..2*n_ff-1 the up rows.
 *  d:   out fp16 bits [n_mat][2*n_ff][ld_d], entries b >= k/32 written as 0.
 *  ld_d: >= k/32, multiple of 8 (use q8_scale_stride(k)).
 * The result equals q8_pack of the row concatenation [gate; up] of every
 * matrix, bit for bit.  qs and d 16-byte aligned; n_ff % 32 == 0.
 */
q8_status q8_pack_up_gate(const float *w_gate, const float *w_up, int64_t n_mat, int64_t n_ff,
                          int64_t k, int8_t *qs, uint16_t *d, int64_t ld_d, void *stream);

/*
 * q8_quantize_row -- Q8_0 activation quantizer ([HADA] 「3段階で構成された修正」:
 * quantize_row_q8_0_x4; the plain one-row form).
 *  x:  fp32 [n_rows][k], 16-byte aligned.  k a multiple of 32, <= Q8_MAX_K.
 *  qs: out int8 [n_rows][k]; d: out fp16 bits [n_rows][k/32] (dense).
 * Bit-exact with the rule in the header comment.
 */
q8_status q8_quantize_row(const float *x, int64_t n_rows, int64_t k, int8_t *qs, uint16_t *d,
                          void *stream);

/*
 * q8_gemv -- y = W x for n_tok quantized activation rows ([NARR]: the Q8_0
 * decode matvec; [HADA] 「非AVX2ビルドで壊れていた演算パス」: the plain Q8_0
 * matrix multiply).
 *  W:   host pointer to a q8_tensor view with n_mat == 1.
 *  xq:  int8 [n_tok][W.k], 16-byte aligned; xd: fp16 bits [n_tok][W.k/32].
 *  n_tok: >= 1.
 *  y:   out fp32 [n_tok][W.rows].
 */
q8_status q8_gemv(const q8_tensor *W, const int8_t *xq, const uint16_t *xd, int64_t n_tok,
                  float *y, void *stream);

/*
 * q8_gemv_batched -- many independent fp32-input GEMVs in one launch.  Each
 * problem quantizes its own x to Q8_0 (the q8_quantize_row rule) and computes
 * y = W x exactly as q8_quantize_row followed by q8_gemv would.
 *  descs: HOST array of n_desc problems (copied into the launch parameters;
 *         the array may be reused as soon as the call returns).
 *  n_desc: 1 .. Q8_MAX_GEMV_DESC.  n_tok: activation rows per problem, >= 1.
 */
typedef struct {
    q8_tensor W;      /* n_mat == 1                                  */
    const float *x;   /* fp32 [n_tok][W.k], 16-byte aligned          */
    float *y;         /* out fp32 [n_tok][W.rows]                    */
} q8_gemv_desc;

q8_status q8_gemv_batched(const q8_gemv_desc *descs, int32_t n_desc, int64_t n_tok,
                          void *stream);

/*
 * Workspace for the routed (MoE) calls: expert grouping tables and the
 * device error word.  ws must be 256-byte aligned; its contents need no
 * initialization.  One workspace may serve consecutive calls on one stream;
 * calls that overlap on the GPU need separate workspaces.
 */
size_t q8_moe_workspace_size(int64_t n_tok, int32_t n_used, int64_t n_mat);

/*
 * q8_moe_up_gate_swiglu -- the fused MoE up/gate + SwiGLU step
 * (MOE_FUSED_UP_GATE; FUSED_UP_GATE when dense).  [HADA]
 * 「非AVX2ビルドで壊れていた演算パス」 and 「3段階で構成された修正」.
 *  up_gate: host pointer to a view with rows == 2*n_ff: in each matrix, rows
 *           0..n_ff-1 are gate and rows n_ff..2*n_ff-1 are up; n_ff % 32 == 0.
 *  xq, xd:  Q8_0 activations [n_tok][k], [n_tok][k/32]; xq 16-byte aligned.
 *  ids:     int32 [n_tok][n_used] expert ids in [0, n_mat), distinct within a
 *           token; or NULL for the dense op (n_mat == 1 and n_used == 1).
 *  For every (t, s), e = ids[t][s], r < n_ff:
 *      g = W_e[r] . x_t,  u = W_e[n_ff + r] . x_t,  h = silu(g) * u,
 *      silu(z) = z / (1 + exp(-z)).
 *  h:   out fp32 [n_tok][n_used][n_ff].
 *  hq, hd: optional (both or neither) out Q8_0 of h: int8 [n_tok][n_used][n_ff],
 *          fp16 bits [n_tok][n_used][n_ff/32]; equal to q8_quantize_row(h).
 *  g_out, u_out: optional fp32 [n_tok][n_used][n_ff] gate and up values.
 *  ws, ws_bytes: required when ids != NULL (see q8_moe_workspace_size).
 */
q8_status q8_moe_up_gate_swiglu(const q8_tensor *up_gate, const int8_t *xq, const uint16_t *xd,
                                int64_t n_tok, const int32_t *ids, int32_t n_used, float *h,
                                int8_t *hq, uint16_t *hd, float *g_out, float *u_out, void *ws,
                                size_t ws_bytes, void *stream);

/*
 * q8_mul_mat_id -- matmul indexed by expert id (ggml_mul_mat_id; [HADA]
 * 「3段階で構成された修正」): y[t][s] = W_{ids[t][s]} . a(t, s).
 *  W:  host pointer to a view (n_mat experts of rows x k).
 *  aq, ad: Q8_0 activations.  a_per_slot != 0: a(t, s) is row t*n_used + s of
 *      [n_tok*n_used][k] (the down projection of h); a_per_slot == 0: a(t, s)
 *      is row t of [n_tok][k] (gate or up slice applied to x).
 *  ids: int32 [n_tok][n_used], required.
 *  y:  out fp32 [n_tok][n_used][W.rows].
 */
q8_status q8_mul_mat_id(const q8_tensor *W, const int8_t *aq, const uint16_t *ad,
                        int32_t a_per_slot, int64_t n_tok, const int32_t *ids, int32_t n_used,
                        float *y, void *ws, size_t ws_bytes, void *stream);

/*
 * q8_moe_group -- the expert grouping that q8_moe_up_gate_swiglu and
 * q8_mul_mat_id run first, as a call of its own: validates ids (errors are
 * latched for q8_check) and writes into ws, for every expert, its count and
 * the list of its pairs p = t*n_used + s in ascending p.  The *_pregrouped
 * calls below then reuse these tables, so one grouping serves the gate/up and
 * the down projection of a layer.
 *  ids: int32 [n_tok][n_used]; ws: q8_moe_workspace_size(n_tok, n_used, n_mat)
 *  bytes, 256-byte aligned.
 */
q8_status q8_moe_group(const int32_t *ids, int64_t n_tok, int32_t n_used, int64_t n_mat,
                       void *ws, size_t ws_bytes, void *stream);

/* q8_moe_up_gate_swiglu on tables written by q8_moe_group for the same
 * (n_tok, n_used, up_gate->n_mat); arguments as in q8_moe_up_gate_swiglu. */
q8_status q8_moe_up_gate_swiglu_pregrouped(const q8_tensor *up_gate, const int8_t *xq,
                                           const uint16_t *xd, int64_t n_tok, int32_t n_used,
                                           float *h, int8_t *hq, uint16_t *hd, float *g_out,
                                           float *u_out, const void *ws, size_t ws_bytes,
                                           void *stream);

/* q8_mul_mat_id on tables written by q8_moe_group for the same
 * (n_tok, n_used, W->n_mat); arguments as in q8_mul_mat_id. */
q8_status q8_mul_mat_id_pregrouped(const q8_tensor *W, const int8_t *aq, const uint16_t *ad,
                                   int32_t a_per_slot, int64_t n_tok, int32_t n_used, float *y,
                                   const void *ws, size_t ws_bytes, void *stream);

/*
 * q8_moe_up_gate_swiglu_fp32 -- q8_moe_up_gate_swiglu for fp32 activations and
 * small batches, with no workspace: each x row is quantized to Q8_0 inside
 * the kernel (bit-exact with q8_quantize_row) and, when ids are given, every
 * CTA groups the routed pairs itself.  One launch.
 *  up_gate: as in q8_moe_up_gate_swiglu.  x: fp32 [n_tok][k], 16-byte aligned.
 *  ids: [n_tok][n_used] or NULL (dense: n_mat == 1, n_used == 1).
 *  Limits: n_tok * n_used <= Q8_SMALL_BATCH_PAIRS, n_mat <= Q8_SMALL_BATCH_MATS
 *  (else Q8_E_UNSUPPORTED: use the workspace calls).
 *  h: out fp32 [n_tok][n_used][n_ff].
 *  err_word: optional device int32; receives the routing-id error flags
 *  (nonzero: an id out of range or repeated in a token; pairs with an
 *  out-of-range id are left unwritten).  Pass the first word of a routed
 *  workspace to have q8_check report them.
 */
#define Q8_SMALL_BATCH_PAIRS 1024
#define Q8_SMALL_BATCH_MATS 512
q8_status q8_moe_up_gate_swiglu_fp32(const q8_tensor *up_gate, const float *x, int64_t n_tok,
                                     const int32_t *ids, int32_t n_used, float *h,
                                     int32_t *err_word, void *stream);

/*
 * q8_mul_mat_id_fp32 -- q8_mul_mat_id for fp32 activations and small
 * batches, with no workspace (activation rows quantized to Q8_0 inside the
 * kernel; routed pairs grouped in every CTA).  Arguments as in
 * q8_mul_mat_id, a: fp32 rows (per slot or per token), 16-byte aligned; the
 * limits and err_word of q8_moe_up_gate_swiglu_fp32.
 */
q8_status q8_mul_mat_id_fp32(const q8_tensor *W, const float *a, int32_t a_per_slot,
                             int64_t n_tok, const int32_t *ids, int32_t n_used, float *y,
                             int32_t *err_word, void *stream);

/*
 * q8_moe_up_gate_swiglu_noalloc -- q8_moe_up_gate_swiglu for callers that
 * cannot allocate device memory (no counterpart on the pages: this is a
 * library convenience, not part of the method).  Some callers cannot call
 * cudaMalloc or an allocating library routine at the point where they run
 * the step: code inside a custom allocator or memory-pool hook, plugins whose
 * host forbids device allocation, or hot loops that must not touch the
 * allocator.  This variant takes no workspace: the expert-grouping tables live
 * in a file-scope device array of Q8_NOALLOC_SCRATCH_BYTES bytes inside
 * libq8, which every GPU that loads the library holds until the process exits.
 *  Arguments, outputs and results are those of q8_moe_up_gate_swiglu (ids
 *  required), except that there is no ws / ws_bytes.
 *  Limit: the grouping tables must fit the scratch, i.e.
 *  q8_moe_workspace_size(n_tok, n_used, up_gate->n_mat) <= Q8_NOALLOC_SCRATCH_BYTES
 *  (for 128 experts and 8 per token: up to 1982 tokens); larger calls return
 *  Q8_E_WORKSPACE and launch nothing.
 *  The first call on each device looks up the scratch address on that device
 *  (cudaGetSymbolAddress, with that device current), and so does the first
 *  call after the device's context was recreated (cudaDeviceReset): the
 *  address is kept per device together with the id of the context it belongs
 *  to.  Make that first call before any stream capture.  Every call shares the one scratch array: calls
 *  that overlap on the GPU (other streams, other host threads) race and give
 *  wrong results; serialize them.  The scratch keeps the last call's contents;
 *  nothing in it needs clearing, because the grouping kernel rewrites every
 *  word that the up/gate kernel later reads.  Routing-id errors are not
 *  reported by this variant (no q8_check): pairs whose id is out of range are
 *  skipped and their outputs left unwritten.
 */
#define Q8_NOALLOC_SCRATCH_BYTES 65536
q8_status q8_moe_up_gate_swiglu_noalloc(const q8_tensor *up_gate, const int8_t *xq,
                                        const uint16_t *xd, int64_t n_tok, const int32_t *ids,
                                        int32_t n_used, float *h, int8_t *hq, uint16_t *hd,
                                        float *g_out, float *u_out, void *stream);

/*
 * q8_moe_combine -- out[t] = sum_{s < n_used} route_w[t][s] * y[t][s], summed in
 * ascending s (the routing-weight combine after the down projection).
 *  y: fp32 [n_tok][n_used][n_out]; route_w: fp32 [n_tok][n_used];
 *  out: fp32 [n_tok][n_out].
 */
q8_status q8_moe_combine(const float *y, const float *route_w, int64_t n_tok, int32_t n_used,
                         int64_t n_out, float *out, void *stream);

/*
 * q8_moe_ffn -- the whole feed-forward step from fp32 x: quantize x, fused
 * up/gate + SwiGLU with h quantized to Q8_0, mul_mat_id down projection and
 * the routing-weight combine.
 *  up_gate: [n_mat][2*n_ff][n_embd] view; down: [n_mat][n_embd][n_ff] view.
 *  x: fp32 [n_tok][n_embd], 16-byte aligned.
 *  ids, route_w: [n_tok][n_used]; both NULL for the dense FFN (n_mat == 1,
 *  n_used == 1), where out = down . quantize(h).
 *  out: fp32 [n_tok][n_embd].
 *  ws: q8_moe_ffn_workspace_size(...) bytes, 256-byte aligned; it also holds
 *      the intermediates (grouping, xq, h, hq, per-slot y) and the grid-barrier
 *      counter of the fused layer kernel, which every fused call advances by
 *      its grid size (the device's SM count).  Zero-fill the workspace before
 *      its first use, use it on one device, and zero it again after a wait
 *      timeout reported by q8_check.  The counter has a fixed place in the
 *      first 256 bytes, which no call of any shape uses for anything else, so
 *      a workspace sized for the largest call serves calls of every smaller
 *      shape in any order.
 * Routed batches of at most 32 pairs (n_tok * n_used) with n_embd <= 4096
 * and n_ff <= 2048 run as ONE cooperative kernel (grouping, up/gate +
 * SwiGLU, a grid barrier, down + combine); the result is bitwise that of
 * the separate calls.  Larger routed batches run quantize + q8_moe_group +
 * q8_moe_up_gate_swiglu_pregrouped (h quantized once) +
 * q8_mul_mat_id_pregrouped + q8_moe_combine, with the same results as those
 * calls.  Dense batches of up to Q8_SMALL_BATCH_PAIRS rows run
 * q8_moe_up_gate_swiglu_fp32 and the down GEMV on fp32 h (n_ff <= 4096) or,
 * for longer h rows, q8_quantize_row of h and q8_gemv (the same bits: the
 * down kernel quantizes h by the same rule).
 */
size_t q8_moe_ffn_workspace_size(int64_t n_tok, int32_t n_used, int64_t n_mat, int64_t n_embd,
                                 int64_t n_ff);
q8_status q8_moe_ffn(const q8_tensor *up_gate, const q8_tensor *down, const float *x,
                     int64_t n_tok, const int32_t *ids, const float *route_w, int32_t n_used,
                     float *out, void *ws, size_t ws_bytes, void *stream);

/*
 * q8_route -- the router, the step before the routed calls: routing ids and
 * routing weights from the activations.  The pages name MoE routing only as
 * a run-time option ([HADA], opening section on the 2016-Xeon set-up:
 * 「CPUを考慮したMoEルーティング」); this is the plain top-k router:
 *    logits[t][e] = sum_i w_router[e][i] * x[t][i], products and sums in fp64;
 *    ids[t]       = the n_used experts with the largest logits, largest first,
 *                   equal logits taken by ascending expert index;
 *    route_w[t]   = softmax over the selected logits only (fp64, stored fp32).
 *  w_router: fp32 [n_exp][n_embd] (not quantized); x: fp32 [n_tok][n_embd];
 *            both 16-byte aligned, n_embd a multiple of 4.
 *  ids: out int32 [n_tok][n_used]; route_w: out fp32 [n_tok][n_used]; they
 *       feed q8_moe_ffn and the other routed calls directly.
 *  logits: optional out fp64 [n_tok][n_exp] (NULL: not written).
 *  Limits: n_exp <= Q8_ROUTE_MAX_EXP, n_used <= min(n_exp, Q8_MAX_USED),
 *  else Q8_E_SHAPE.  NaN logits rank as -infinity.
 * One launch of thread-block clusters (8 CTAs per group of up to 4 tokens,
 * fewer when one token's fp64 activations and logits, 8 * n_embd + 8 *
 * n_exp bytes, leave no room for more; the experts split
 * across the cluster, the top-k read through distributed shared memory).
 */
#define Q8_ROUTE_MAX_EXP 1024
q8_status q8_route(const float *w_router, const float *x, int64_t n_tok, int64_t n_embd,
                   int64_t n_exp, int32_t n_used, int32_t *ids, float *route_w, double *logits,
                   void *stream);

/*
 * q8_check -- synchronize `stream` and report errors found on the device:
 *  - Q8_E_BAD_ID if ws (optional; NULL skips this check) holds a routing-id
 *    error from the last routed call that used it: an id out of range or
 *    repeated within a token.  The outputs of pairs with out-of-range ids are
 *    then unspecified.
 *  - Q8_E_CUDA if the stream reported an error, or if a kernel on this
 *    device gave up waiting (after about 2 s) for a shared-memory stage or
 *    for the other CTAs of its grid; that flag stays set until
 *    q8_reset_errors clears it, and results computed since it was set are
 *    not to be trusted.
 * Else Q8_OK.
 */
q8_status q8_check(const void *ws, void *stream);

/*
 * q8_reset_errors -- clear the wait-timeout flags (the Q8_E_CUDA condition
 * of q8_check above) on the current device, so that one timeout does not
 * poison every later check.  Synchronous; call it while no libq8 kernel is
 * running on the device.  Routing-id errors live in the caller's workspace
 * and are rewritten by every routed call; they need no reset.  After a
 * timeout inside q8_moe_ffn's fused layer kernel, also zero that call's
 * workspace (its grid-barrier words are left inconsistent).
 */
q8_status q8_reset_errors(void);

/*
 * q8_debug_wait_timeout -- test hook for the bounded waits: runs one wait
 * that cannot succeed, which gives up after limit_ns nanoseconds, latches the
 * wait-timeout flag that q8_check reports and returns (the kernel ends; the
 * device stays usable).
 *  kind 0: an mbarrier wait on a phase that nothing completes (the wait of
 *          every streaming kernel's shared-memory ring).
 *  kind 1: the fused layer kernel's grid barrier with one arrival short; bar
 *          is a device pointer to a zeroed, 8-byte aligned 64-bit counter,
 *          which the call leaves off its multiple.
 *  limit_ns: 1e3 .. 1e10.
 * Clear the flag afterwards with q8_reset_errors.
 */
q8_status q8_debug_wait_timeout(int32_t kind, int64_t limit_ns, unsigned *bar, void *stream);

/*
 * q8_debug_block_dots -- test hook: the exact int32 per-block dots of the
 * given weight rows of matrix `mat` with one activation row, through the same
 * device dot-product routine the matmul kernels use.
 *  rows: device int64 [n_rows] row indices; isum: out int32 [n_rows][W.k/32].
 */
q8_status q8_debug_block_dots(const q8_tensor *W, int64_t mat, const int64_t *rows,
                              int64_t n_rows, const int8_t *xq, int32_t *isum, void *stream);

/* Text for a status code (static storage). */
const char *q8_status_string(q8_status s);

/* Detail text of the last non-OK status returned on this host thread. */
const char *q8_last_error(void);

#ifdef __cplusplus
}
#endif

#endif /* Q8_H */
