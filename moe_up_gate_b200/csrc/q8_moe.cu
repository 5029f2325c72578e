// q8_moe.cu -- the routed (MoE) part of libq8: expert grouping, the fused
// up/gate + SwiGLU kernel (with h quantized to Q8_0 in its epilogue), the
// routing-weight combine and the whole feed-forward step.
//
// The op is MOE_FUSED_UP_GATE / FUSED_UP_GATE of the news.hada.io article on
// Gemma 4 26B-A4B Q8_0 (sections 「非AVX2ビルドで壊れていた演算パス」 and
// 「3段階で構成された修正」): per routed expert, gate and up rows from one
// combined weight whose first half is gate and second half up, then
// silu(gate) * up.  Where the article's fallback runs two mul_mat_id over two
// view_3d slices and a separate fused_mul_unary, this kernel reads gate row r
// and up row n_ff + r in the same pass and applies SwiGLU in registers.
#include <algorithm>
#include <mutex>

#include "q8_internal.h"
#include "q8_tile.cuh"

namespace q8 {

constexpr int kThreadsMoe = 256;

// ---------------------------------------------------------------------------
// Expert grouping: one CTA.  Validates ids (range, repeats within a token),
// counts pairs per expert, writes offsets (exclusive scan), the ascending
// lists of experts with pairs (split at big_threshold) and the pairs sorted
// by expert then by pair index (a stable counting sort: one warp walks the
// pairs in order, 32 at a time, ranking equal experts with __match_any_sync).
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(1024) group_kernel(const int32_t *__restrict__ ids, int n_tok,
                                                     int n_used, int n_mat, int big_threshold,
                                                     int32_t *__restrict__ ws, GroupLayout L) {
    extern __shared__ int sm_group[];
    int *cnt = sm_group;
    int *cursor = sm_group + n_mat;
    __shared__ int s_err;
    const int P = n_tok * n_used;
    for (int e = threadIdx.x; e < n_mat; e += blockDim.x) cnt[e] = 0;
    if (threadIdx.x == 0) s_err = 0;
    __syncthreads();
    int err = 0;
    for (int p = threadIdx.x; p < P; p += blockDim.x) {
        const int e = ids[p];
        if (e < 0 || e >= n_mat) {
            err |= ERR_ID_RANGE;
            continue;
        }
        atomicAdd(&cnt[e], 1);
        const int t = p / n_used;
        const int s = p - t * n_used;
        for (int s2 = 0; s2 < s; ++s2)
            if (ids[t * n_used + s2] == e) err |= ERR_ID_REPEAT;
    }
    if (err) atomicOr(&s_err, err);
    __syncthreads();
    const int lane = threadIdx.x & 31;
    if (threadIdx.x < 32) {
        int running = 0, n_small = 0, n_big = 0;
        for (int base = 0; base < n_mat; base += 32) {
            const int e = base + lane;
            const int c = e < n_mat ? cnt[e] : 0;
            int incl = c;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const int v = __shfl_up_sync(0xffffffffu, incl, o);
                if (lane >= o) incl += v;
            }
            const int off = running + incl - c;
            if (e < n_mat) {
                ws[L.count + e] = c;
                ws[L.offset + e] = off;
                cursor[e] = off;
            }
            const bool small = c > 0 && c < big_threshold;
            const bool big = c >= big_threshold && c > 0;
            const unsigned bs = __ballot_sync(0xffffffffu, small);
            const unsigned bb = __ballot_sync(0xffffffffu, big);
            const unsigned lt = (1u << lane) - 1u;
            if (small) ws[L.list_small + n_small + __popc(bs & lt)] = e;
            if (big) ws[L.list_big + n_big + __popc(bb & lt)] = e;
            n_small += __popc(bs);
            n_big += __popc(bb);
            running += __shfl_sync(0xffffffffu, incl, 31);
        }
        if (lane == 0) {
            ws[L.offset + n_mat] = running;
            ws[WS_ERR] = s_err;
            ws[WS_N_SMALL] = n_small;
            ws[WS_N_BIG] = n_big;
            ws[WS_N_PAIRS] = P;
        }
        __syncwarp();
        // stable scatter of the valid pairs
        for (int base = 0; base < P; base += 32) {
            const int p = base + lane;
            const int e = p < P ? ids[p] : -1;
            const bool valid = e >= 0 && e < n_mat;
            const int key = valid ? e : n_mat + lane;  // invalid lanes match nobody
            const unsigned m = __match_any_sync(0xffffffffu, key);
            const int rank = __popc(m & ((1u << lane) - 1u));
            if (valid) ws[L.pairs + cursor[e] + rank] = p;
            __syncwarp();
            if (valid && (__ffs(m) - 1) == lane) cursor[e] += __popc(m);
            __syncwarp();
        }
    }
}

q8_status launch_group(const int32_t *ids, int64_t n_tok, int32_t n_used, int64_t n_mat,
                       int32_t big_threshold, int32_t *ws, cudaStream_t s) {
    const GroupLayout L = group_layout(n_tok * n_used, n_mat);
    const size_t smem = (size_t)2 * n_mat * sizeof(int);
    group_kernel<<<1, 1024, smem, s>>>(ids, (int)n_tok, n_used, (int)n_mat, big_threshold, ws, L);
    return launch_status("group_kernel");
}

// ---------------------------------------------------------------------------
// Fused up/gate + SwiGLU.  CTA (tile, slot): gate rows [32*tile, 32*tile+32)
// of expert e (the slot-th expert of the grouping list, or matrix 0 when
// dense) and the matching up rows n_ff + r, for every pair routed to e, NT
// pairs at a time.  Each warp takes G gate rows and their G up rows in one
// streaming pass (2G rows through dot_rows).  The 32 h values of a pair form
// exactly one Q8_0 block of h, quantized in the epilogue.
// ---------------------------------------------------------------------------
struct UpGateParams {
    const int8_t *wq;
    const uint16_t *wd;
    int64_t ld_d;
    int64_t mat_stride;
    int k;
    int n_ff;
    const int8_t *xq;
    const uint16_t *xd;
    float *h;
    int8_t *hq;
    uint16_t *hd;
    float *g_out;
    float *u_out;
    const int32_t *ws;
    int64_t lay_count, lay_offset, lay_list, lay_pairs;
    int list_word;
    int n_dense;
    int n_used;
};

__device__ __forceinline__ float silu_f(float z) { return z / (1.0f + expf(-z)); }

template <int NT, int G>
__global__ void __launch_bounds__(kThreadsMoe) up_gate_kernel(const UpGateParams p) {
    extern __shared__ __align__(16) unsigned char smem[];
    __shared__ int s_pair[NT];
    __shared__ int s_arow[NT];
    __shared__ float s_h[NT][32];
    const int nb = p.k / QK;
    int e = 0, cnt = p.n_dense;
    const int32_t *plist = nullptr;
    if (p.ws) {
        if ((int)blockIdx.y >= p.ws[p.list_word]) return;
        e = p.ws[p.lay_list + blockIdx.y];
        cnt = p.ws[p.lay_count + e];
        plist = p.ws + p.lay_pairs + p.ws[p.lay_offset + e];
    }
    const int lane = threadIdx.x & 31;
    const int warp = threadIdx.x >> 5;
    const int nwarps = blockDim.x >> 5;
    const int tile = blockIdx.x;
    const int r_base = tile * 32;
    const int8_t *wq = p.wq + (int64_t)e * p.mat_stride * p.k;
    const uint16_t *wd = p.wd + (int64_t)e * p.mat_stride * p.ld_d;
    const XStage xs = make_xstage(smem, NT, nb);
    for (int pg = 0; pg < cnt; pg += NT) {
        const int n = min(NT, cnt - pg);
        if ((int)threadIdx.x < n) {
            const int pr = plist ? plist[pg + threadIdx.x] : pg + (int)threadIdx.x;
            s_pair[threadIdx.x] = pr;
            s_arow[threadIdx.x] = p.ws ? pr / p.n_used : pr;
        }
        __syncthreads();
        stage_q8_rows(xs, p.xq, p.xd, p.k, s_arow, n);
        __syncthreads();
        for (int gg = warp * G; gg < 32; gg += nwarps * G) {
            const int8_t *wrow[2 * G];
            const uint16_t *drow[2 * G];
#pragma unroll
            for (int j = 0; j < G; ++j) {
                const int64_t rg = r_base + gg + j;
                const int64_t ru = p.n_ff + rg;
                wrow[j] = wq + rg * p.k;
                drow[j] = wd + rg * p.ld_d;
                wrow[G + j] = wq + ru * p.k;
                drow[G + j] = wd + ru * p.ld_d;
            }
            float acc[2 * G][NT];
#pragma unroll
            for (int r = 0; r < 2 * G; ++r)
#pragma unroll
                for (int t = 0; t < NT; ++t) acc[r][t] = 0.0f;
            dot_rows<NT, 2 * G>(wrow, drow, xs, n, lane, acc);
            reduce_rows<NT, 2 * G>(acc);
#pragma unroll
            for (int j = 0; j < G; ++j)
#pragma unroll
                for (int t = 0; t < NT; ++t)
                    if (lane == ((j * NT + t) & 31) && t < n) {
                        const float g = acc[j][t];
                        const float u = acc[G + j][t];
                        const float hv = silu_f(g) * u;
                        const int64_t o = (int64_t)s_pair[t] * p.n_ff + r_base + gg + j;
                        p.h[o] = hv;
                        s_h[t][gg + j] = hv;
                        if (p.g_out) p.g_out[o] = g;
                        if (p.u_out) p.u_out[o] = u;
                    }
        }
        __syncthreads();
        if (p.hq) {
            for (int t = warp; t < n; t += nwarps) {
                const float v = s_h[t][lane];
                const float amax = warp_max_all(fabsf(v));
                const float d32 = block_scale(amax);
                const float id = block_inv_scale(d32);
                const int64_t pr = s_pair[t];
                p.hq[pr * p.n_ff + r_base + lane] = (int8_t)quantize_one(v, id);
                if (lane == 0) p.hd[pr * (p.n_ff / QK) + tile] = scale_bits(d32);
            }
        }
        __syncthreads();
    }
}

static int pick_nt_moe(int64_t max_group) {
    if (max_group <= 1) return 1;
    if (max_group <= 2) return 2;
    if (max_group <= 4) return 4;
    return 8;
}

static q8_status launch_up_gate(const UpGateParams &p, int64_t max_group, int64_t slots,
                                cudaStream_t s) {
    const int nt = pick_nt_moe(max_group);
    const dim3 grid((unsigned)(p.n_ff / 32), (unsigned)slots);
    const size_t smem = (size_t)nt * xstage_bytes_per_row(p.k / QK);
#define Q8_LAUNCH_UG(NT_, G_)                                                                \
    do {                                                                                     \
        if (smem > 48 * 1024)                                                                \
            cudaFuncSetAttribute(up_gate_kernel<NT_, G_>,                                    \
                                 cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);     \
        up_gate_kernel<NT_, G_><<<grid, kThreadsMoe, smem, s>>>(p);                          \
    } while (0)
    switch (nt) {
        case 1: Q8_LAUNCH_UG(1, 4); break;
        case 2: Q8_LAUNCH_UG(2, 2); break;
        case 4: Q8_LAUNCH_UG(4, 2); break;
        default: Q8_LAUNCH_UG(8, 1); break;
    }
#undef Q8_LAUNCH_UG
    return launch_status("up_gate_kernel");
}

// ---------------------------------------------------------------------------
// Combine: out[t][r] = sum_s w[t][s] * y[t][s][r], s ascending (fma chain).
// ---------------------------------------------------------------------------
__global__ void combine_kernel(const float *__restrict__ y, const float *__restrict__ w,
                               int n_tok, int n_used, int n_out, float *__restrict__ out) {
    const int64_t total = (int64_t)n_tok * n_out;
    for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < total;
         i += (int64_t)gridDim.x * blockDim.x) {
        const int64_t t = i / n_out;
        const int64_t r = i - t * n_out;
        float acc = 0.0f;
        for (int s = 0; s < n_used; ++s)
            acc = fmaf(w[t * n_used + s], y[(t * n_used + s) * n_out + r], acc);
        out[i] = acc;
    }
}

static q8_status launch_combine(const float *y, const float *w, int64_t n_tok, int32_t n_used,
                                int64_t n_out, float *out, cudaStream_t s) {
    const int64_t total = n_tok * n_out;
    const int blocks = (int)std::min<int64_t>((total + 255) / 256, 148 * 8);
    combine_kernel<<<blocks, 256, 0, s>>>(y, w, (int)n_tok, n_used, (int)n_out, out);
    return launch_status("combine_kernel");
}

// moe_ffn workspace regions
struct FfnLayout {
    size_t group, xq, xd, h, hq, hd, y, total;
};

static FfnLayout ffn_layout(int64_t n_tok, int32_t n_used, int64_t n_mat, int64_t n_embd,
                            int64_t n_ff, bool routed) {
    FfnLayout L{};
    const int64_t P = n_tok * n_used;
    size_t o = 0;
    L.group = o;
    o += routed ? group_bytes(P, n_mat) : 0;
    L.xq = o;
    o += round_up((size_t)n_tok * n_embd, 256);
    L.xd = o;
    o += round_up((size_t)n_tok * (n_embd / QK) * 2, 256);
    L.h = o;
    o += round_up((size_t)P * n_ff * 4, 256);
    L.hq = o;
    o += round_up((size_t)P * n_ff, 256);
    L.hd = o;
    o += round_up((size_t)P * (n_ff / QK) * 2, 256);
    L.y = o;
    o += routed ? round_up((size_t)P * n_embd * 4, 256) : 0;
    L.total = o;
    return L;
}

}  // namespace q8

using namespace q8;

extern "C" {

size_t q8_moe_workspace_size(int64_t n_tok, int32_t n_used, int64_t n_mat) {
    if (n_tok < 1 || n_used < 1 || n_mat < 1) return 0;
    return group_bytes(n_tok * n_used, n_mat);
}

// Shared body of the routed/dense up_gate entry points.  group: run the
// grouping kernel on ids first (else the tables in ws are reused).
static q8_status up_gate_entry(const char *fn, const q8_tensor *up_gate, const int8_t *xq,
                               const uint16_t *xd, int64_t n_tok, const int32_t *ids,
                               bool routed, bool group, int32_t n_used, float *h, int8_t *hq,
                               uint16_t *hd, float *g_out, float *u_out, const void *ws,
                               size_t ws_bytes, cudaStream_t s) {
    q8_status st = check_tensor(up_gate, fn, false);
    if (st != Q8_OK) return st;
    Q8_REQUIRE(xq && xd && h, Q8_E_NULL, "%s: NULL pointer", fn);
    Q8_REQUIRE((hq == nullptr) == (hd == nullptr), Q8_E_NULL, "%s: hq and hd go together", fn);
    Q8_REQUIRE(up_gate->rows % 64 == 0, Q8_E_SHAPE,
               "%s: rows=%lld must be 2*n_ff with n_ff %% 32 == 0", fn, (long long)up_gate->rows);
    Q8_REQUIRE(n_tok >= 1 && n_used >= 1 && n_used <= Q8_MAX_USED &&
                   n_tok * n_used <= (1LL << 24),
               Q8_E_SHAPE, "%s: n_tok=%lld n_used=%d", fn, (long long)n_tok, n_used);
    Q8_REQUIRE(aligned16(xq), Q8_E_ALIGN, "%s: xq must be 16-byte aligned", fn);
    const int64_t n_ff = up_gate->rows / 2;
    UpGateParams p{};
    p.wq = up_gate->qs;
    p.wd = up_gate->d;
    p.ld_d = up_gate->ld_d;
    p.mat_stride = up_gate->mat_stride;
    p.k = (int)up_gate->k;
    p.n_ff = (int)n_ff;
    p.xq = xq;
    p.xd = xd;
    p.h = h;
    p.hq = hq;
    p.hd = hd;
    p.g_out = g_out;
    p.u_out = u_out;
    p.n_used = n_used;
    if (!routed) {
        Q8_REQUIRE(up_gate->n_mat == 1 && n_used == 1, Q8_E_SHAPE,
                   "%s: dense call (ids NULL) needs n_mat == 1, n_used == 1", fn);
        p.ws = nullptr;
        p.n_dense = (int)n_tok;
        return launch_up_gate(p, n_tok, 1, s);
    }
    Q8_REQUIRE(up_gate->n_mat <= 4096, Q8_E_UNSUPPORTED, "%s: n_mat > 4096", fn);
    Q8_REQUIRE(ws != nullptr && aligned256(ws), Q8_E_WORKSPACE,
               "%s: workspace NULL or not 256-byte aligned", fn);
    Q8_REQUIRE(ws_bytes >= q8_moe_workspace_size(n_tok, n_used, up_gate->n_mat), Q8_E_WORKSPACE,
               "%s: workspace too small", fn);
    const int64_t P = n_tok * n_used;
    if (group) {
        st = launch_group(ids, n_tok, n_used, up_gate->n_mat, 1 << 30, (int32_t *)ws, s);
        if (st != Q8_OK) return st;
    }
    const GroupLayout L = group_layout(P, up_gate->n_mat);
    p.ws = (const int32_t *)ws;
    p.lay_count = L.count;
    p.lay_offset = L.offset;
    p.lay_list = L.list_small;
    p.lay_pairs = L.pairs;
    p.list_word = WS_N_SMALL;
    return launch_up_gate(p, n_tok, std::min<int64_t>(up_gate->n_mat, P), s);
}

q8_status q8_moe_up_gate_swiglu(const q8_tensor *up_gate, const int8_t *xq, const uint16_t *xd,
                                int64_t n_tok, const int32_t *ids, int32_t n_used, float *h,
                                int8_t *hq, uint16_t *hd, float *g_out, float *u_out, void *ws,
                                size_t ws_bytes, void *stream) {
    return up_gate_entry("q8_moe_up_gate_swiglu", up_gate, xq, xd, n_tok, ids, ids != nullptr,
                         true, n_used, h, hq, hd, g_out, u_out, ws, ws_bytes,
                         (cudaStream_t)stream);
}

q8_status q8_moe_up_gate_swiglu_pregrouped(const q8_tensor *up_gate, const int8_t *xq,
                                           const uint16_t *xd, int64_t n_tok, int32_t n_used,
                                           float *h, int8_t *hq, uint16_t *hd, float *g_out,
                                           float *u_out, const void *ws, size_t ws_bytes,
                                           void *stream) {
    return up_gate_entry("q8_moe_up_gate_swiglu_pregrouped", up_gate, xq, xd, n_tok, nullptr,
                         true, false, n_used, h, hq, hd, g_out, u_out, ws, ws_bytes,
                         (cudaStream_t)stream);
}

// ---------------------------------------------------------------------------
// Allocation-free variant: the grouping tables live in this file-scope device
// array instead of a caller workspace.  Host code must not pass the array's
// name to a kernel (on the host it is only a stand-in symbol); its device
// address is looked up once per device with cudaGetSymbolAddress.
// ---------------------------------------------------------------------------
static __device__ __align__(256) int32_t g_noalloc_scratch[Q8_NOALLOC_SCRATCH_BYTES / 4];

constexpr int kMaxDevices = 64;
static std::mutex g_noalloc_mu;
static void *g_noalloc_addr[kMaxDevices] = {};

static q8_status noalloc_scratch_address(void **out) {
    int dev = -1;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess)
        Q8_FAIL(Q8_E_CUDA, "q8_moe_up_gate_swiglu_noalloc: cudaGetDevice: %s",
                cudaGetErrorString(e));
    Q8_REQUIRE(dev >= 0 && dev < kMaxDevices, Q8_E_UNSUPPORTED,
               "q8_moe_up_gate_swiglu_noalloc: device %d beyond %d", dev, kMaxDevices);
    std::lock_guard<std::mutex> lock(g_noalloc_mu);
    if (g_noalloc_addr[dev] == nullptr) {
        void *p = nullptr;
        e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
        if (e != cudaSuccess || p == nullptr)
            Q8_FAIL(Q8_E_CUDA, "q8_moe_up_gate_swiglu_noalloc: cudaGetSymbolAddress: %s",
                    cudaGetErrorString(e));
        g_noalloc_addr[dev] = p;
    }
    *out = g_noalloc_addr[dev];
    return Q8_OK;
}

q8_status q8_moe_group(const int32_t *ids, int64_t n_tok, int32_t n_used, int64_t n_mat,
                       void *ws, size_t ws_bytes, void *stream) {
    Q8_REQUIRE(ids != nullptr, Q8_E_NULL, "q8_moe_group: ids is NULL");
    Q8_REQUIRE(n_tok >= 1 && n_used >= 1 && n_used <= Q8_MAX_USED &&
                   n_tok * n_used <= (1LL << 24) && n_mat >= 1,
               Q8_E_SHAPE, "q8_moe_group: n_tok=%lld n_used=%d n_mat=%lld", (long long)n_tok,
               n_used, (long long)n_mat);
    Q8_REQUIRE(n_mat <= 4096, Q8_E_UNSUPPORTED, "q8_moe_group: n_mat > 4096");
    Q8_REQUIRE(((uintptr_t)ids & 3u) == 0, Q8_E_ALIGN, "q8_moe_group: ids misaligned");
    Q8_REQUIRE(ws != nullptr && aligned256(ws), Q8_E_WORKSPACE,
               "q8_moe_group: workspace NULL or not 256-byte aligned");
    Q8_REQUIRE(ws_bytes >= q8_moe_workspace_size(n_tok, n_used, n_mat), Q8_E_WORKSPACE,
               "q8_moe_group: workspace too small");
    return launch_group(ids, n_tok, n_used, n_mat, 1 << 30, (int32_t *)ws, (cudaStream_t)stream);
}

q8_status q8_moe_up_gate_swiglu_noalloc(const q8_tensor *up_gate, const int8_t *xq,
                                        const uint16_t *xd, int64_t n_tok, const int32_t *ids,
                                        int32_t n_used, float *h, int8_t *hq, uint16_t *hd,
                                        float *g_out, float *u_out, void *stream) {
    const char *fn = "q8_moe_up_gate_swiglu_noalloc";
    Q8_REQUIRE(up_gate != nullptr && ids != nullptr, Q8_E_NULL, "%s: up_gate and ids required",
               fn);
    Q8_REQUIRE(n_tok >= 1 && n_used >= 1 && n_used <= Q8_MAX_USED &&
                   n_tok * n_used <= (1LL << 24) && up_gate->n_mat >= 1,
               Q8_E_SHAPE, "%s: n_tok=%lld n_used=%d", fn, (long long)n_tok, n_used);
    const size_t need = q8_moe_workspace_size(n_tok, n_used, up_gate->n_mat);
    Q8_REQUIRE(need <= (size_t)Q8_NOALLOC_SCRATCH_BYTES, Q8_E_WORKSPACE,
               "%s: n_tok*n_used=%lld with n_mat=%lld needs %zu bytes of grouping scratch; the "
               "built-in scratch holds %d (use q8_moe_up_gate_swiglu with a workspace)",
               fn, (long long)(n_tok * n_used), (long long)up_gate->n_mat, need,
               Q8_NOALLOC_SCRATCH_BYTES);
    void *scratch = nullptr;
    q8_status st = noalloc_scratch_address(&scratch);
    if (st != Q8_OK) return st;
    return up_gate_entry(fn, up_gate, xq, xd, n_tok, ids, true, true, n_used, h, hq, hd, g_out,
                         u_out, scratch, Q8_NOALLOC_SCRATCH_BYTES, (cudaStream_t)stream);
}

q8_status q8_moe_combine(const float *y, const float *route_w, int64_t n_tok, int32_t n_used,
                         int64_t n_out, float *out, void *stream) {
    Q8_REQUIRE(y && route_w && out, Q8_E_NULL, "q8_moe_combine: NULL pointer");
    Q8_REQUIRE(n_tok >= 1 && n_used >= 1 && n_used <= Q8_MAX_USED && n_out >= 1 &&
                   n_out < (1LL << 31),
               Q8_E_SHAPE, "q8_moe_combine: bad sizes");
    return launch_combine(y, route_w, n_tok, n_used, n_out, out, (cudaStream_t)stream);
}

size_t q8_moe_ffn_workspace_size(int64_t n_tok, int32_t n_used, int64_t n_mat, int64_t n_embd,
                                 int64_t n_ff) {
    if (n_tok < 1 || n_used < 1 || n_mat < 1 || n_embd < 32 || n_ff < 32) return 0;
    return ffn_layout(n_tok, n_used, n_mat, n_embd, n_ff, true).total;
}

q8_status q8_moe_ffn(const q8_tensor *up_gate, const q8_tensor *down, const float *x,
                     int64_t n_tok, const int32_t *ids, const float *route_w, int32_t n_used,
                     float *out, void *ws, size_t ws_bytes, void *stream) {
    q8_status st = check_tensor(up_gate, "q8_moe_ffn: up_gate", false);
    if (st != Q8_OK) return st;
    st = check_tensor(down, "q8_moe_ffn: down", false);
    if (st != Q8_OK) return st;
    Q8_REQUIRE(x && out, Q8_E_NULL, "q8_moe_ffn: NULL pointer");
    Q8_REQUIRE((ids == nullptr) == (route_w == nullptr), Q8_E_NULL,
               "q8_moe_ffn: ids and route_w go together");
    const int64_t n_embd = up_gate->k;
    const int64_t n_ff = up_gate->rows / 2;
    Q8_REQUIRE(up_gate->rows % 64 == 0, Q8_E_SHAPE, "q8_moe_ffn: up_gate rows must be 2*n_ff, "
               "n_ff %% 32 == 0");
    Q8_REQUIRE(down->k == n_ff && down->rows == n_embd && down->n_mat == up_gate->n_mat,
               Q8_E_SHAPE, "q8_moe_ffn: down must be [n_mat][n_embd][n_ff]");
    Q8_REQUIRE(n_tok >= 1 && n_used >= 1 && n_used <= Q8_MAX_USED &&
                   n_tok * n_used <= (1LL << 24),
               Q8_E_SHAPE, "q8_moe_ffn: n_tok=%lld n_used=%d", (long long)n_tok, n_used);
    Q8_REQUIRE(aligned16(x), Q8_E_ALIGN, "q8_moe_ffn: x must be 16-byte aligned");
    const bool routed = ids != nullptr;
    if (!routed)
        Q8_REQUIRE(up_gate->n_mat == 1 && n_used == 1, Q8_E_SHAPE,
                   "q8_moe_ffn: dense call needs n_mat == 1 and n_used == 1");
    else
        Q8_REQUIRE(up_gate->n_mat <= 4096, Q8_E_UNSUPPORTED, "q8_moe_ffn: n_mat > 4096");
    const FfnLayout F = ffn_layout(n_tok, n_used, up_gate->n_mat, n_embd, n_ff, routed);
    Q8_REQUIRE(ws != nullptr && aligned256(ws), Q8_E_WORKSPACE,
               "q8_moe_ffn: workspace NULL or not 256-byte aligned");
    Q8_REQUIRE(ws_bytes >= F.total, Q8_E_WORKSPACE, "q8_moe_ffn: workspace too small");
    cudaStream_t s = (cudaStream_t)stream;
    unsigned char *w8 = (unsigned char *)ws;
    int8_t *xq = (int8_t *)(w8 + F.xq);
    uint16_t *xd = (uint16_t *)(w8 + F.xd);
    float *h = (float *)(w8 + F.h);
    int8_t *hq = (int8_t *)(w8 + F.hq);
    uint16_t *hd = (uint16_t *)(w8 + F.hd);
    st = q8_quantize_row(x, n_tok, n_embd, xq, xd, s);
    if (st != Q8_OK) return st;
    if (!routed) {
        st = q8_moe_up_gate_swiglu(up_gate, xq, xd, n_tok, nullptr, 1, h, hq, hd, nullptr, nullptr,
                                   nullptr, 0, s);
        if (st != Q8_OK) return st;
        return q8_gemv(down, hq, hd, n_tok, out, s);
    }
    int32_t *wsg = (int32_t *)(w8 + F.group);
    const size_t gbytes = group_bytes(n_tok * n_used, up_gate->n_mat);
    // one grouping serves the gate/up and the down projection
    st = q8_moe_group(ids, n_tok, n_used, up_gate->n_mat, wsg, gbytes, s);
    if (st != Q8_OK) return st;
    st = q8_moe_up_gate_swiglu_pregrouped(up_gate, xq, xd, n_tok, n_used, h, hq, hd, nullptr,
                                          nullptr, wsg, gbytes, s);
    if (st != Q8_OK) return st;
    float *y = (float *)(w8 + F.y);
    st = q8_mul_mat_id_pregrouped(down, hq, hd, 1, n_tok, n_used, y, wsg, gbytes, s);
    if (st != Q8_OK) return st;
    return launch_combine(y, route_w, n_tok, n_used, n_embd, out, s);
}

q8_status q8_check(const void *ws, void *stream) {
    Q8_REQUIRE(ws != nullptr, Q8_E_NULL, "q8_check: ws is NULL");
    cudaStream_t s = (cudaStream_t)stream;
    int32_t flags = 0;
    cudaError_t e = cudaMemcpyAsync(&flags, ws, sizeof flags, cudaMemcpyDeviceToHost, s);
    if (e == cudaSuccess) e = cudaStreamSynchronize(s);
    if (e != cudaSuccess) Q8_FAIL(Q8_E_CUDA, "q8_check: %s", cudaGetErrorString(e));
    if (flags & ERR_ID_RANGE) Q8_FAIL(Q8_E_BAD_ID, "q8_check: a routing id is out of range");
    if (flags & ERR_ID_REPEAT)
        Q8_FAIL(Q8_E_BAD_ID, "q8_check: a routing id repeats within a token");
    return Q8_OK;
}

}  // extern "C"
