// q8_matmul.cu -- Q8_0 x Q8_0 matrix-vector kernels: the batch-1 GEMV
// (q8_gemv), many independent GEMVs in one launch (q8_gemv_batched) and the
// matmul indexed by expert id (q8_mul_mat_id), plus the block-dot test hook.
//
// The Q8_0 decode matvec is the hot loop of the Llama 2 110M int8 decode in
// the "narray-llm" README (section "Llama 2 110M を int8 (Q8_0) で");
// mul_mat_id is ggml_mul_mat_id of the news.hada.io article (section
// 「3段階で構成された修正」), applied per routed expert.
#include <algorithm>

#include "q8_internal.h"
#include "q8_tile.cuh"

namespace q8 {

constexpr int kThreads = 256;

// ---------------------------------------------------------------------------
// matmul over a group of activation rows per matrix.
//   dense  (ws == nullptr): matrix 0, pairs 0..n_dense-1, activation row = pair.
//   routed (ws != nullptr): CTA row blockIdx.y is the blockIdx.y-th expert of
//     the grouping list; its pairs come from the grouping tables; activation
//     row = pair (a_per_slot) or pair / n_used.
// Output y[pair][row].
// ---------------------------------------------------------------------------
struct MatmulParams {
    const int8_t *wq;
    const uint16_t *wd;
    int64_t ld_d;
    int64_t mat_stride;
    int k;
    int rows;
    const int8_t *aq;
    const uint16_t *ad;
    float *y;
    const int32_t *ws;
    int64_t lay_count, lay_offset, lay_list, lay_pairs;
    int list_word;  // WS_N_SMALL or WS_N_BIG
    int n_dense;
    int a_per_slot;
    int n_used;
    int rows_per_cta;
};

template <int NT, int R>
__global__ void __launch_bounds__(kThreads) matmul_kernel(const MatmulParams p) {
    extern __shared__ __align__(16) unsigned char smem[];
    __shared__ int s_pair[NT];
    __shared__ int s_arow[NT];
    const int nb = p.k / QK;
    int e = 0, cnt = p.n_dense;
    const int32_t *plist = nullptr;
    if (p.ws) {
        if ((int)blockIdx.y >= p.ws[p.list_word]) return;
        e = p.ws[p.lay_list + blockIdx.y];
        cnt = p.ws[p.lay_count + e];
        plist = p.ws + p.lay_pairs + p.ws[p.lay_offset + e];
    }
    const int row0 = blockIdx.x * p.rows_per_cta;
    const int row_end = min(p.rows, row0 + p.rows_per_cta);
    const int8_t *wq = p.wq + (int64_t)e * p.mat_stride * p.k;
    const uint16_t *wd = p.wd + (int64_t)e * p.mat_stride * p.ld_d;
    const XStage xs = make_xstage(smem, NT, nb);
    for (int pg = 0; pg < cnt; pg += NT) {
        const int n = min(NT, cnt - pg);
        if ((int)threadIdx.x < n) {
            const int pr = plist ? plist[pg + threadIdx.x] : pg + (int)threadIdx.x;
            s_pair[threadIdx.x] = pr;
            s_arow[threadIdx.x] = (!p.ws || p.a_per_slot) ? pr : pr / p.n_used;
        }
        __syncthreads();
        stage_q8_rows(xs, p.aq, p.ad, p.k, s_arow, n);
        __syncthreads();
        run_rows<NT, R>(wq, wd, p.k, p.ld_d, p.rows, row0, row_end, xs, n, s_pair, p.y);
        __syncthreads();
    }
}

static int pick_nt(int64_t max_rows_per_group) {
    if (max_rows_per_group <= 1) return 1;
    if (max_rows_per_group <= 2) return 2;
    if (max_rows_per_group <= 4) return 4;
    return 8;
}

// Rows per CTA: enough CTAs to cover the SMs several times over, in whole
// warp row groups.
static int pick_rows_per_cta(int64_t rows, int64_t slots, int R) {
    const int64_t unit = (int64_t)(kThreads / 32) * R;
    int64_t rpc = unit * 4;
    while (rpc > unit && ((rows + rpc - 1) / rpc) * slots < 4 * 148) rpc -= unit;
    return (int)rpc;
}

q8_status launch_matmul(const MatmulParams &base, int64_t max_group, int64_t slots,
                        cudaStream_t s) {
    MatmulParams p = base;
    const int nt = pick_nt(max_group);
    const int R = (nt <= 2) ? 4 : 2;
    p.rows_per_cta = pick_rows_per_cta(p.rows, slots, R);
    const dim3 grid((unsigned)((p.rows + p.rows_per_cta - 1) / p.rows_per_cta), (unsigned)slots);
    const size_t smem = (size_t)nt * xstage_bytes_per_row(p.k / QK);
#define Q8_LAUNCH_MM(NT_, R_)                                                                \
    do {                                                                                     \
        if (smem > 48 * 1024)                                                                \
            cudaFuncSetAttribute(matmul_kernel<NT_, R_>,                                     \
                                 cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);     \
        matmul_kernel<NT_, R_><<<grid, kThreads, smem, s>>>(p);                              \
    } while (0)
    switch (nt) {
        case 1: Q8_LAUNCH_MM(1, 4); break;
        case 2: Q8_LAUNCH_MM(2, 4); break;
        case 4: Q8_LAUNCH_MM(4, 2); break;
        default: Q8_LAUNCH_MM(8, 2); break;
    }
#undef Q8_LAUNCH_MM
    return launch_status("matmul_kernel");
}

// ---------------------------------------------------------------------------
// Batched GEMV: independent problems, fp32 inputs quantized in the CTA.
// ---------------------------------------------------------------------------
struct GemvProblem {
    const int8_t *wq;
    const uint16_t *wd;
    const float *x;
    float *y;
    int64_t ld_d;
    int k;
    int rows;
    int rows_per_cta;
    int tile_begin;
};

struct GemvBatchParams {
    int n_desc;
    int n_tok;
    int total_tiles;
    int max_nb;
    GemvProblem pr[Q8_MAX_GEMV_DESC];
};

template <int NT, int R>
__global__ void __launch_bounds__(kThreads) gemv_batched_kernel(const __grid_constant__ GemvBatchParams p) {
    extern __shared__ __align__(16) unsigned char smem[];
    __shared__ int s_pair[NT];
    // which problem does this tile belong to (tile_begin is increasing)
    int lo = 0, hi = p.n_desc - 1;
    while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (p.pr[mid].tile_begin <= (int)blockIdx.x) lo = mid; else hi = mid - 1;
    }
    const GemvProblem &q = p.pr[lo];
    const int tile = blockIdx.x - q.tile_begin;
    const int row0 = tile * q.rows_per_cta;
    const int row_end = min(q.rows, row0 + q.rows_per_cta);
    const XStage xs = make_xstage(smem, NT, q.k / QK);
    for (int pg = 0; pg < p.n_tok; pg += NT) {
        const int n = min(NT, p.n_tok - pg);
        if ((int)threadIdx.x < n) s_pair[threadIdx.x] = pg + threadIdx.x;
        stage_f32_rows(xs, q.x + (int64_t)pg * q.k, q.k, n);
        __syncthreads();
        run_rows<NT, R>(q.wq, q.wd, q.k, q.ld_d, q.rows, row0, row_end, xs, n, s_pair, q.y);
        __syncthreads();
    }
}

// ---------------------------------------------------------------------------
// Test hook: per-block int32 dots through block_dot.
// ---------------------------------------------------------------------------
// A row index outside [0, n_w_rows) writes INT32_MIN for each of its blocks
// and reads nothing.
__global__ void block_dots_kernel(const int8_t *__restrict__ wq, int k, int64_t n_w_rows,
                                  const int64_t *rows, int64_t n_rows,
                                  const int8_t *__restrict__ xq, int32_t *__restrict__ isum) {
    const int nb = k / QK;
    const int64_t total = n_rows * nb;
    for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < total;
         i += (int64_t)gridDim.x * blockDim.x) {
        const int64_t ri = i / nb;
        const int kb = (int)(i - ri * nb);
        const int64_t row = rows[ri];
        if (row < 0 || row >= n_w_rows) {
            isum[i] = INT32_MIN;
            continue;
        }
        const int8_t *w = wq + row * k + kb * QK;
        const int8_t *x = xq + kb * QK;
        const uint4 w0 = *reinterpret_cast<const uint4 *>(w);
        const uint4 w1 = *reinterpret_cast<const uint4 *>(w + 16);
        const uint4 x0 = *reinterpret_cast<const uint4 *>(x);
        const uint4 x1 = *reinterpret_cast<const uint4 *>(x + 16);
        isum[i] = block_dot(w0, w1, x0, x1);
    }
}

// mul_mat_id over grouping tables already written to ws by launch_group.
q8_status launch_matmul_routed(const q8_tensor *W, const int8_t *aq, const uint16_t *ad,
                               int a_per_slot, int64_t n_tok, int32_t n_used, float *y,
                               const int32_t *ws, cudaStream_t s) {
    const int64_t P = n_tok * n_used;
    const GroupLayout L = group_layout(P, W->n_mat);
    MatmulParams p{};
    p.wq = W->qs;
    p.wd = W->d;
    p.ld_d = W->ld_d;
    p.mat_stride = W->mat_stride;
    p.k = (int)W->k;
    p.rows = (int)W->rows;
    p.aq = aq;
    p.ad = ad;
    p.y = y;
    p.ws = ws;
    p.lay_count = L.count;
    p.lay_offset = L.offset;
    p.lay_list = L.list_small;
    p.lay_pairs = L.pairs;
    p.list_word = WS_N_SMALL;
    p.a_per_slot = a_per_slot ? 1 : 0;
    p.n_used = n_used;
    const int64_t slots = std::min<int64_t>(W->n_mat, P);
    return launch_matmul(p, n_tok, slots, s);
}

}  // namespace q8

using namespace q8;

extern "C" {

q8_status q8_gemv(const q8_tensor *W, const int8_t *xq, const uint16_t *xd, int64_t n_tok,
                  float *y, void *stream) {
    q8_status st = check_tensor(W, "q8_gemv: W", true);
    if (st != Q8_OK) return st;
    Q8_REQUIRE(xq && xd && y, Q8_E_NULL, "q8_gemv: NULL pointer");
    Q8_REQUIRE(n_tok >= 1 && n_tok <= (1 << 20), Q8_E_SHAPE, "q8_gemv: n_tok=%lld",
               (long long)n_tok);
    Q8_REQUIRE(W->rows < (1LL << 31), Q8_E_SHAPE, "q8_gemv: rows too large");
    Q8_REQUIRE(aligned16(xq), Q8_E_ALIGN, "q8_gemv: xq must be 16-byte aligned");
    Q8_REQUIRE(((uintptr_t)xd & 1u) == 0 && ((uintptr_t)y & 3u) == 0, Q8_E_ALIGN,
               "q8_gemv: xd/y misaligned");
    MatmulParams p{};
    p.wq = W->qs;
    p.wd = W->d;
    p.ld_d = W->ld_d;
    p.mat_stride = W->mat_stride;
    p.k = (int)W->k;
    p.rows = (int)W->rows;
    p.aq = xq;
    p.ad = xd;
    p.y = y;
    p.ws = nullptr;
    p.n_dense = (int)n_tok;
    return launch_matmul(p, n_tok, 1, (cudaStream_t)stream);
}

static q8_status mul_mat_id_entry(const char *fn, const q8_tensor *W, const int8_t *aq,
                                  const uint16_t *ad, int32_t a_per_slot, int64_t n_tok,
                                  const int32_t *ids, bool group, int32_t n_used, float *y,
                                  const void *ws, size_t ws_bytes, cudaStream_t s) {
    q8_status st = check_tensor(W, fn, false);
    if (st != Q8_OK) return st;
    Q8_REQUIRE(aq && ad && y && (ids || !group), Q8_E_NULL, "%s: NULL pointer", fn);
    Q8_REQUIRE(n_tok >= 1 && n_used >= 1 && n_used <= Q8_MAX_USED &&
                   n_tok * n_used <= (1LL << 24),
               Q8_E_SHAPE, "%s: n_tok=%lld n_used=%d", fn, (long long)n_tok, n_used);
    Q8_REQUIRE(W->n_mat <= 4096, Q8_E_UNSUPPORTED, "%s: n_mat > 4096", fn);
    Q8_REQUIRE(W->rows < (1LL << 31), Q8_E_SHAPE, "%s: rows too large", fn);
    Q8_REQUIRE(aligned16(aq), Q8_E_ALIGN, "%s: aq must be 16-byte aligned", fn);
    Q8_REQUIRE(((uintptr_t)ad & 1u) == 0 && ((uintptr_t)y & 3u) == 0 &&
                   ((uintptr_t)ids & 3u) == 0,
               Q8_E_ALIGN, "%s: ad/y/ids misaligned", fn);
    Q8_REQUIRE(ws != nullptr && aligned256(ws), Q8_E_WORKSPACE,
               "%s: workspace NULL or not 256-byte aligned", fn);
    Q8_REQUIRE(ws_bytes >= q8_moe_workspace_size(n_tok, n_used, W->n_mat), Q8_E_WORKSPACE,
               "%s: workspace too small", fn);
    if (group) {
        st = launch_group(ids, n_tok, n_used, W->n_mat, 1 << 30, (int32_t *)ws, s);
        if (st != Q8_OK) return st;
    }
    return launch_matmul_routed(W, aq, ad, a_per_slot, n_tok, n_used, y, (const int32_t *)ws, s);
}

q8_status q8_mul_mat_id(const q8_tensor *W, const int8_t *aq, const uint16_t *ad,
                        int32_t a_per_slot, int64_t n_tok, const int32_t *ids, int32_t n_used,
                        float *y, void *ws, size_t ws_bytes, void *stream) {
    return mul_mat_id_entry("q8_mul_mat_id", W, aq, ad, a_per_slot, n_tok, ids, true, n_used, y,
                            ws, ws_bytes, (cudaStream_t)stream);
}

q8_status q8_mul_mat_id_pregrouped(const q8_tensor *W, const int8_t *aq, const uint16_t *ad,
                                   int32_t a_per_slot, int64_t n_tok, int32_t n_used, float *y,
                                   const void *ws, size_t ws_bytes, void *stream) {
    return mul_mat_id_entry("q8_mul_mat_id_pregrouped", W, aq, ad, a_per_slot, n_tok, nullptr,
                            false, n_used, y, ws, ws_bytes, (cudaStream_t)stream);
}

q8_status q8_gemv_batched(const q8_gemv_desc *descs, int32_t n_desc, int64_t n_tok,
                          void *stream) {
    Q8_REQUIRE(descs != nullptr, Q8_E_NULL, "q8_gemv_batched: descs is NULL");
    Q8_REQUIRE(n_desc >= 1 && n_desc <= Q8_MAX_GEMV_DESC, Q8_E_SHAPE,
               "q8_gemv_batched: n_desc=%d", n_desc);
    Q8_REQUIRE(n_tok >= 1 && n_tok <= 4096, Q8_E_SHAPE, "q8_gemv_batched: n_tok=%lld",
               (long long)n_tok);
    static_assert(sizeof(GemvBatchParams) < 32000, "kernel parameter block too large");
    GemvBatchParams p{};
    p.n_desc = n_desc;
    p.n_tok = (int)n_tok;
    const int nt = pick_nt(n_tok);
    const int R = (nt <= 2) ? 4 : 2;
    int tiles = 0, max_nb = 0;
    int64_t total_rows = 0;
    for (int i = 0; i < n_desc; ++i) total_rows += descs[i].W.rows;
    for (int i = 0; i < n_desc; ++i) {
        const q8_gemv_desc &d = descs[i];
        q8_status st = check_tensor(&d.W, "q8_gemv_batched: W", true);
        if (st != Q8_OK) return st;
        Q8_REQUIRE(d.x && d.y, Q8_E_NULL, "q8_gemv_batched: problem %d x/y NULL", i);
        Q8_REQUIRE(aligned16(d.x) && ((uintptr_t)d.y & 3u) == 0, Q8_E_ALIGN,
                   "q8_gemv_batched: problem %d x must be 16-byte aligned", i);
        Q8_REQUIRE(d.W.rows < (1LL << 31), Q8_E_SHAPE, "q8_gemv_batched: rows too large");
        GemvProblem &q = p.pr[i];
        q.wq = d.W.qs;
        q.wd = d.W.d;
        q.x = d.x;
        q.y = d.y;
        q.ld_d = d.W.ld_d;
        q.k = (int)d.W.k;
        q.rows = (int)d.W.rows;
        // equal weight bytes per CTA across problems: ~16 KB, whole warp row groups
        const int unit = (kThreads / 32) * R;
        int rpc = (int)std::max<int64_t>(unit, (16384 / d.W.k) / unit * unit);
        q.rows_per_cta = rpc;
        q.tile_begin = tiles;
        tiles += (int)((d.W.rows + rpc - 1) / rpc);
        max_nb = std::max(max_nb, (int)(d.W.k / QK));
    }
    p.total_tiles = tiles;
    p.max_nb = max_nb;
    const size_t smem = (size_t)nt * xstage_bytes_per_row(max_nb);
    cudaStream_t s = (cudaStream_t)stream;
#define Q8_LAUNCH_GB(NT_, R_)                                                                \
    do {                                                                                     \
        if (smem > 48 * 1024)                                                                \
            cudaFuncSetAttribute(gemv_batched_kernel<NT_, R_>,                               \
                                 cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);     \
        gemv_batched_kernel<NT_, R_><<<tiles, kThreads, smem, s>>>(p);                       \
    } while (0)
    switch (nt) {
        case 1: Q8_LAUNCH_GB(1, 4); break;
        case 2: Q8_LAUNCH_GB(2, 4); break;
        case 4: Q8_LAUNCH_GB(4, 2); break;
        default: Q8_LAUNCH_GB(8, 2); break;
    }
#undef Q8_LAUNCH_GB
    return launch_status("gemv_batched_kernel");
}

q8_status q8_debug_block_dots(const q8_tensor *W, int64_t mat, const int64_t *rows,
                              int64_t n_rows, const int8_t *xq, int32_t *isum, void *stream) {
    q8_status st = check_tensor(W, "q8_debug_block_dots: W", false);
    if (st != Q8_OK) return st;
    Q8_REQUIRE(rows && xq && isum, Q8_E_NULL, "q8_debug_block_dots: NULL pointer");
    Q8_REQUIRE(mat >= 0 && mat < W->n_mat, Q8_E_SHAPE, "q8_debug_block_dots: mat out of range");
    Q8_REQUIRE(n_rows >= 1, Q8_E_SHAPE, "q8_debug_block_dots: n_rows < 1");
    Q8_REQUIRE(aligned16(xq), Q8_E_ALIGN, "q8_debug_block_dots: xq must be 16-byte aligned");
    const int8_t *wq = W->qs + mat * W->mat_stride * W->k;
    const int64_t total = n_rows * (W->k / QK);
    const int blocks = (int)std::min<int64_t>((total + 255) / 256, 1024);
    block_dots_kernel<<<blocks, 256, 0, (cudaStream_t)stream>>>(wq, (int)W->k, W->rows, rows,
                                                                n_rows, xq, isum);
    return launch_status("block_dots_kernel");
}

}  // extern "C"
