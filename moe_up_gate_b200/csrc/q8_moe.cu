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
#include "q8_stream.cuh"

namespace q8 {

// ---------------------------------------------------------------------------
// Expert grouping: one CTA.  Validates ids (range, repeats within a token),
// counts pairs per expert, writes offsets (exclusive scan), the ascending
// lists of experts with pairs (split at big_threshold) and the pairs sorted
// by expert then by pair index (a stable counting sort: one warp walks the
// pairs in order, 32 at a time, ranking equal experts with __match_any_sync).
// When they fit (staged), the ids are read from global memory once, by all
// threads, into shared memory, so the checks and the warp's walk read them
// there.
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(1024) group_kernel(const int32_t *__restrict__ ids, int n_tok,
                                                     int n_used, int n_mat, int big_threshold,
                                                     int staged, int32_t *__restrict__ ws,
                                                     GroupLayout L) {
    extern __shared__ int sm_group[];
    int *cnt = sm_group;
    int *cursor = sm_group + n_mat;
    int *sid = sm_group + 2 * n_mat;  // the ids, when staged
    __shared__ int s_err;
    const int P = n_tok * n_used;
    griddep_wait();  // ids may come from, and ws may still be read by, earlier kernels
    griddep_launch_dependents();
    for (int e = threadIdx.x; e < n_mat; e += blockDim.x) cnt[e] = 0;
    if (staged)
        for (int p = threadIdx.x; p < P; p += blockDim.x) sid[p] = ids[p];
    if (threadIdx.x == 0) s_err = 0;
    __syncthreads();
    const int32_t *idv = staged ? sid : ids;
    int err = 0;
    for (int p = threadIdx.x; p < P; p += blockDim.x) {
        const int e = idv[p];
        if (e < 0 || e >= n_mat) {
            err |= ERR_ID_RANGE;
            continue;
        }
        atomicAdd(&cnt[e], 1);
        const int t = p / n_used;
        const int s = p - t * n_used;
        for (int s2 = 0; s2 < s; ++s2)
            if (idv[t * n_used + s2] == e) err |= ERR_ID_REPEAT;
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
    }
    __syncthreads();
    const unsigned lt = (1u << lane) - 1u;
    if (staged == 2) {
        // stable scatter by all 32 warps: warp w takes the pairs of its
        // contiguous segment; its base for expert e is the expert's offset
        // plus the pairs of e in the segments before it (counted per warp
        // first, then summed over the warps in order)
        const int warp = threadIdx.x >> 5;
        int *wc = sid + P + warp * n_mat;  // this warp's counts, then bases
        const int per = ((P + 31) / 32 + 31) / 32 * 32;
        const int p0 = min(P, warp * per), p1 = min(P, p0 + per);
        for (int e = lane; e < n_mat; e += 32) wc[e] = 0;
        __syncwarp();
        for (int base = p0; base < p1; base += 32) {
            const int p = base + lane;
            const int e = p < p1 ? idv[p] : -1;
            const bool valid = e >= 0 && e < n_mat;
            const unsigned m = __match_any_sync(0xffffffffu, valid ? e : n_mat + lane);
            if (valid && (m & lt) == 0u) wc[e] += __popc(m);
            __syncwarp();
        }
        __syncthreads();
        for (int e = threadIdx.x; e < n_mat; e += blockDim.x) {
            int run = cursor[e];
            for (int w2 = 0; w2 < 32; ++w2) {
                const int c = sid[P + w2 * n_mat + e];
                sid[P + w2 * n_mat + e] = run;
                run += c;
            }
        }
        __syncthreads();
        for (int base = p0; base < p1; base += 32) {
            const int p = base + lane;
            const int e = p < p1 ? idv[p] : -1;
            const bool valid = e >= 0 && e < n_mat;
            const unsigned m = __match_any_sync(0xffffffffu, valid ? e : n_mat + lane);
            if (valid) ws[L.pairs + wc[e] + __popc(m & lt)] = p;
            __syncwarp();
            if (valid && (m & lt) == 0u) wc[e] += __popc(m);
            __syncwarp();
        }
    } else if (threadIdx.x < 32) {
        // stable scatter of the valid pairs by one warp, 32 at a time
        for (int base = 0; base < P; base += 32) {
            const int p = base + lane;
            const int e = p < P ? idv[p] : -1;
            const bool valid = e >= 0 && e < n_mat;
            const int key = valid ? e : n_mat + lane;  // invalid lanes match nobody
            const unsigned m = __match_any_sync(0xffffffffu, key);
            const int rank = __popc(m & lt);
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
    const int64_t P = n_tok * n_used;
    // counts and cursors (n_mat <= 4096: at most 32 KB), then the ids when the
    // whole stays inside the 48 KB a launch gets without an opt-in
    const int64_t base = 2 * n_mat * (int64_t)sizeof(int);
    const int64_t ids_bytes = P * (int64_t)sizeof(int);
    const int64_t warp_bytes = 32 * n_mat * (int64_t)sizeof(int);  // per-warp counts
    // 2: ids and per-warp counts fit and there are pairs enough for every
    // warp (all warps scatter; 256 tokens of the 128-expert layer: 4.7%
    // faster per layer); 1: ids fit (one warp scatters); 0: neither
    const int staged = P >= 512 && base + ids_bytes + warp_bytes + 256 <= 48 * 1024 ? 2
                       : base + ids_bytes + 256 <= 48 * 1024      ? 1
                                                                   : 0;
    const size_t smem = (size_t)(base + (staged ? ids_bytes : 0) + (staged == 2 ? warp_bytes : 0));
    return launch_pdl("group_kernel", group_kernel, dim3(1), dim3(1024), smem, s, ids, (int)n_tok,
                      n_used, (int)n_mat, big_threshold, staged, ws, L);
}

// Wait timeouts of the kernels in this file (read by q8_check).
static __device__ int g_err_moe;

q8_status read_wait_errors_moe(int *flags) {
    cudaError_t e = cudaMemcpyFromSymbol(flags, g_err_moe, sizeof(int));
    return e == cudaSuccess ? Q8_OK : Q8_E_CUDA;
}

q8_status clear_wait_errors_moe() {
    const int zero = 0;
    cudaError_t e = cudaMemcpyToSymbol(g_err_moe, &zero, sizeof(int));
    return e == cudaSuccess ? Q8_OK : Q8_E_CUDA;
}

// ---------------------------------------------------------------------------
// Fused up/gate + SwiGLU on the streaming engine.  A tile is nr/2 gate rows
// [r0, r0 + nr/2) of one expert and the matching up rows n_ff + r0 ..., both
// streamed into one stage (gate rows first, up rows from stage row nr/2), so
// one pass over the combined weight yields g and u of every routed pair of
// that expert; the epilogue applies h = silu(g) * u in registers.
// Dense (ws == nullptr): matrix 0, activation rows = pairs 0..n_dense-1.
// Routed: the experts of the grouping list; activation row of pair p is
// p / n_used (every slot of a token reads the token's x).
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
    const float *xf;  // fp32 x instead of xq/xd (quantized while staged)
    float *h;
    float *g_out;
    float *u_out;
    const int32_t *ws;
    int64_t lay_count, lay_offset, lay_list, lay_pairs, lay_big;
    int include_big;  // the dp4a kernel also takes the tensor-core list
    int n_dense;
    int n_used;
    // routed with the grouping built in each CTA from ids (ws unused)
    const int32_t *ids;
    int n_tok;
    int n_mat;
    int32_t *err_out;
    Plan plan;
};

__device__ __forceinline__ float silu_f(float z) { return z / (1.0f + expf(-z)); }

// Dense: an instantiation for dense calls (no grouping table, no ids), whose
// activation staging takes the wide form (stage_f32).
template <int NT, bool Dense>
__global__ void __launch_bounds__(kThreadsStream, ctas_per_sm(NT))
    up_gate_kernel(const __grid_constant__ UpGateParams p) {
    extern __shared__ __align__(128) unsigned char smem[];
    Q8_TRACE(0);
    const Ring R = ring_init(smem, p.plan);
    Q8_TRACE(1);
    const Geo g = geo_pair_for_k(p.k);
    const int half_rows = g.nr / 2;
    const int tpm = p.n_ff / half_rows;
    griddep_launch_dependents();
    const int32_t *tab = Dense ? nullptr : p.ws;
    if (!Dense && p.ids) {
        griddep_wait();
        int32_t *stab = reinterpret_cast<int32_t *>(smem + p.plan.off_tab);
        GroupLayout L{};
        L.count = p.lay_count;
        L.offset = p.lay_offset;
        L.list_small = p.lay_list;
        L.list_big = p.lay_big;
        L.pairs = p.lay_pairs;
        cta_group(p.ids, p.n_tok, p.n_used, p.n_mat, L, stab, p.err_out);
        tab = stab;
        Q8_TRACE(3);
    } else if (tab) {
        griddep_wait();
    }
    const bool routed = tab != nullptr;
    const int n_small = routed ? tab[WS_N_SMALL] : 1;
    const int n_mat = n_small + ((routed && p.include_big) ? tab[WS_N_BIG] : 0);
    auto expert = [&](int mi) {
        return mi < n_small ? tab[p.lay_list + mi] : tab[p.lay_big + (mi - n_small)];
    };
    int64_t tb, te;
    my_tiles((int64_t)n_mat * tpm, &tb, &te);
    if ((threadIdx.x >> 5) == kCW) {  // producer warp
        if ((threadIdx.x & 31) == 0 && tb < te) {
            auto src = [&](int64_t t) {
                TileSrc ts{};
                const int mi = (int)(t / tpm), ti = (int)(t % tpm);
                const int e = routed ? expert(mi) : 0;
                const int64_t gate_row = (int64_t)e * p.mat_stride + (int64_t)ti * half_rows;
                const int64_t up_row = gate_row + p.n_ff;
                ts.q0 = p.wq + gate_row * p.k;
                ts.d0 = p.wd + gate_row * p.ld_d;
                ts.rows0 = half_rows;
                ts.q1 = p.wq + up_row * p.k;
                ts.d1 = p.wd + up_row * p.ld_d;
                ts.rows1 = half_rows;
                ts.row_off1 = half_rows;
                ts.k = p.k;
                ts.ld_d = (int)p.ld_d;
                return ts;
            };
            if (p.xf && R.raw_rows > 0) {
                XJobs J;
                const int xmax = p.plan.xmax;
                auto jobs = [&](int64_t t, int when) {
                    const int mi = (int)(t / tpm);
                    const int e = routed ? expert(mi) : 0;
                    const int cnt = routed ? tab[p.lay_count + e] : p.n_dense;
                    const int32_t *plist = routed ? tab + p.lay_pairs + tab[p.lay_offset + e] : nullptr;
                    const int n_grp = (cnt + xmax - 1) / xmax;
                    for (int grp = when; grp < (when == 0 ? min(1, n_grp) : n_grp); ++grp) {
                        const int x0 = grp * xmax;
                        produce_job(R, J, mi, grp, min(xmax, cnt - x0), p.k, [&](int j) {
                            const int pr = plist ? plist[x0 + j] : x0 + j;
                            return p.xf + (int64_t)(routed ? pr / p.n_used : pr) * p.k;
                        }, &g_err_moe);
                    }
                };
                produce(R, tb, te, src, &g_err_moe, jobs, !routed);
            } else {
                produce(R, tb, te, src, &g_err_moe);
            }
        }
        return;
    }
    if (!routed) griddep_wait();
    Q8_TRACE(2);
    const XStage xs{reinterpret_cast<int8_t *>(smem + p.plan.off_xq),
                    reinterpret_cast<float *>(smem + p.plan.off_xd)};
    float *part0 = reinterpret_cast<float *>(smem + p.plan.off_part);
    const int xmax = p.plan.xmax;
    int buf = 0, staged_mi = -1, staged_grp = -1, it = 0;
    XJobs J;
    for (int64_t t = tb; t < te; ++t, ++it) {
        const int s = it % R.stages;
        mbar_wait(&R.full[s], (it / R.stages) & 1, &g_err_moe);
        Q8_TRACE(6);
        const int mi = (int)(t / tpm), ti = (int)(t % tpm);
        const int e = routed ? expert(mi) : 0;
        const int cnt = routed ? tab[p.lay_count + e] : p.n_dense;
        const int32_t *plist = routed ? tab + p.lay_pairs + tab[p.lay_offset + e] : nullptr;
        const int r0 = ti * half_rows;
        const int n_grp = (cnt + xmax - 1) / xmax;
        if (n_grp == 0) {
            __syncwarp();
            if ((threadIdx.x & 31) == 0) mbar_arrive(&R.empty[s]);
        }
        for (int grp = 0; grp < n_grp; ++grp) {
            const int x0 = grp * xmax;
            const int nx = min(xmax, cnt - x0);
            if (mi != staged_mi || grp != staged_grp) {
                // after passes without a barrier every warp must be done
                // with the staged rows before they are replaced
                if (g.wpr == 1 && staged_mi >= 0) named_bar_sync(kBarConsumers, kCT);
                auto arow = [&](int j) {
                    const int pr = plist ? plist[x0 + j] : x0 + j;
                    return routed ? pr / p.n_used : pr;
                };
                if (p.xf)
                    stage_job_f32<Dense>(R, J, xs, p.xf, p.k, nx, arow, &g_err_moe);
                else
                    stage_q8(xs, p.xq, p.xd, p.k, nx, arow);
                named_bar_sync(kBarConsumers, kCT);
                Q8_TRACE(7);
                staged_mi = mi;
                staged_grp = grp;
            }
            for (int tg = 0; tg < nx; tg += NT) {
                const int n = min(NT, nx - tg);
                float *part = part0 + buf * kPartRows * NT;
                with_nt<NT>(n, [&](auto ntc) {
                    constexpr int NTC = decltype(ntc)::value;
                    if (g.wpr == 1) {
                        // whole rows per warp: each warp forms h of its rows
                        warp_pairs<NTC>(R.qs(s), R.d(s), p.k, (int)p.ld_d, g, half_rows, xs, tg,
                                        n, [&](int row, int tt, float gv, float uv) {
                                            if (tt < n) {
                                                const int pr = plist ? plist[x0 + tg + tt]
                                                                     : x0 + tg + tt;
                                                const int64_t o = (int64_t)pr * p.n_ff + r0 + row;
                                                p.h[o] = silu_f(gv) * uv;
                                                if (p.g_out) p.g_out[o] = gv;
                                                if (p.u_out) p.u_out[o] = uv;
                                            }
                                        });
                        Q8_TRACE(8);
                        if (grp == n_grp - 1 && tg + NT >= nx) {
                            __syncwarp();
                            if ((threadIdx.x & 31) == 0) mbar_arrive(&R.empty[s]);
                        }
                        return;
                    }
                    warp_rows_to_part<NTC>(R.qs(s), R.d(s), p.k, (int)p.ld_d, g, xs, tg, n, part);
                    Q8_TRACE(8);
                    if (grp == n_grp - 1 && tg + NT >= nx) {
                        __syncwarp();
                        if ((threadIdx.x & 31) == 0) mbar_arrive(&R.empty[s]);
                    }
                    named_bar_sync(kBarConsumers, kCT);
                    Q8_TRACE(9);
                    for (int i = threadIdx.x; i < half_rows * n; i += kCT) {
                        const int row = i / n;
                        const int tt = i - row * n;
                        const int pr = plist ? plist[x0 + tg + tt] : x0 + tg + tt;
                        const float gv = part_sum<NTC>(part, g, row, tt);
                        const float uv = part_sum<NTC>(part, g, row + half_rows, tt);
                        const int64_t o = (int64_t)pr * p.n_ff + r0 + row;
                        p.h[o] = silu_f(gv) * uv;
                        if (p.g_out) p.g_out[o] = gv;
                        if (p.u_out) p.u_out[o] = uv;
                    }
                    Q8_TRACE(10);
                });
                buf ^= 1;
            }
        }
    }
}

static q8_status launch_up_gate(const UpGateParams &base, RowPlan rp, int64_t slots,
                                cudaStream_t s) {
    UpGateParams p = base;
    const int nt = pick_nt(rp.nt_rows);
    const int tab_words =
        p.ids ? (int)group_layout((int64_t)p.n_tok * p.n_used, p.n_mat).words : 0;
    int tq, td;
    tile_bytes(geo_pair_for_k(p.k), p.k, p.ld_d, &tq, &td);
    if (!make_plan(tq, td, p.k, (int)std::min<int64_t>(rp.x_rows, kMaxXRows), nt, &p.plan,
                   tab_words, p.xf != nullptr && aligned16(p.xf)))
        Q8_FAIL(Q8_E_UNSUPPORTED, "up_gate: k=%d does not fit the shared-memory plan", p.k);
    const Geo g = geo_pair_for_k(p.k);
    const int64_t tiles = slots * (p.n_ff / (g.nr / 2));
    const int grid = (int)std::max<int64_t>(1, std::min<int64_t>((int64_t)num_sms() * p.plan.ctas, tiles));
    if (!p.ids && !p.ws) {
        switch (nt) {
            case 1: return launch_stream(up_gate_kernel<1, true>, grid, p.plan.bytes, s, p, "up_gate");
            case 2: return launch_stream(up_gate_kernel<2, true>, grid, p.plan.bytes, s, p, "up_gate");
            case 4: return launch_stream(up_gate_kernel<4, true>, grid, p.plan.bytes, s, p, "up_gate");
            default: return launch_stream(up_gate_kernel<8, true>, grid, p.plan.bytes, s, p, "up_gate");
        }
    }
    switch (nt) {
        case 1: return launch_stream(up_gate_kernel<1, false>, grid, p.plan.bytes, s, p, "up_gate");
        case 2: return launch_stream(up_gate_kernel<2, false>, grid, p.plan.bytes, s, p, "up_gate");
        case 4: return launch_stream(up_gate_kernel<4, false>, grid, p.plan.bytes, s, p, "up_gate");
        default: return launch_stream(up_gate_kernel<8, false>, grid, p.plan.bytes, s, p, "up_gate");
    }
}

// ---------------------------------------------------------------------------
// Combine: out[t][r] = sum_s w[t][s] * y[t][s][r], s ascending (fma chain).
// ---------------------------------------------------------------------------
__global__ void combine_kernel(const float *__restrict__ y, const float *__restrict__ w,
                               int n_tok, int n_used, int n_out, float *__restrict__ out) {
    griddep_wait();
    griddep_launch_dependents();
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

// The same sums, four outputs per thread (n_out a multiple of 4, 16-byte
// aligned rows; fewer than 2^31 outputs): 16-byte loads and stores, 32-bit
// indices, the slots' loads issued eight at a time.
__global__ void combine4_kernel(const float4 *__restrict__ y, const float *__restrict__ w,
                                int n_tok, int n_used, int n_out4, float4 *__restrict__ out) {
    griddep_wait();
    griddep_launch_dependents();
    const int total = n_tok * n_out4;
    for (int i = blockIdx.x * blockDim.x + threadIdx.x; i < total; i += gridDim.x * blockDim.x) {
        const int t = i / n_out4;
        const int r = i - t * n_out4;
        float4 acc = make_float4(0.0f, 0.0f, 0.0f, 0.0f);
#pragma unroll 8
        for (int s = 0; s < n_used; ++s) {
            const float ws = w[t * n_used + s];
            const float4 v = y[(t * n_used + s) * n_out4 + r];
            acc.x = fmaf(ws, v.x, acc.x);
            acc.y = fmaf(ws, v.y, acc.y);
            acc.z = fmaf(ws, v.z, acc.z);
            acc.w = fmaf(ws, v.w, acc.w);
        }
        out[i] = acc;
    }
}

static q8_status launch_combine(const float *y, const float *w, int64_t n_tok, int32_t n_used,
                                int64_t n_out, float *out, cudaStream_t s) {
    const int64_t total = n_tok * n_out;
    if (n_out % 4 == 0 && aligned16(y) && aligned16(out) &&
        (int64_t)n_tok * n_used * n_out < ((int64_t)1 << 31)) {
        const int64_t total4 = total / 4;
        const int blocks = (int)std::min<int64_t>((total4 + 255) / 256, 148 * 8);
        return launch_pdl("combine_kernel", combine4_kernel, dim3((unsigned)blocks), dim3(256), 0,
                          s, reinterpret_cast<const float4 *>(y), w, (int)n_tok, n_used,
                          (int)(n_out / 4), reinterpret_cast<float4 *>(out));
    }
    const int blocks = (int)std::min<int64_t>((total + 255) / 256, 148 * 8);
    return launch_pdl("combine_kernel", combine_kernel, dim3((unsigned)blocks), dim3(256), 0, s, y,
                      w, (int)n_tok, n_used, (int)n_out, out);
}

// moe_ffn workspace regions.  The grouping region comes first and always
// holds at least its header, whose words WS_BAR.. are the fused layer
// kernel's grid-barrier words: a fixed place that no shape-dependent region
// of any call overlaps.
struct FfnLayout {
    size_t group, xq, xd, h, hq, hd, y, total;
};

static FfnLayout ffn_layout(int64_t n_tok, int32_t n_used, int64_t n_mat, int64_t n_embd,
                            int64_t n_ff, bool routed) {
    FfnLayout L{};
    const int64_t P = n_tok * n_used;
    size_t o = 0;
    L.group = o;
    o += routed ? group_bytes(P, n_mat) : 256;
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
    p.g_out = g_out;
    p.u_out = u_out;
    p.n_used = n_used;
    if (!routed) {
        Q8_REQUIRE(up_gate->n_mat == 1 && n_used == 1, Q8_E_SHAPE,
                   "%s: dense call (ids NULL) needs n_mat == 1, n_used == 1", fn);
        p.ws = nullptr;
        p.n_dense = (int)n_tok;
        if (n_tok >= kTcMinDense && n_tok <= kTcMaxDense && tc_eligible(up_gate, true) && !g_out &&
            !u_out)
            st = launch_tc(up_gate, true, xq, xd, nullptr, 1, n_tok, 1, h, nullptr, s);
        else
            st = launch_up_gate(p, dense_rows(n_tok), 1, s);
        if (st != Q8_OK || hq == nullptr) return st;
        // h -> Q8_0 with the activation quantizer (a 32-block of h spans
        // several weight tiles, so it is not formed inside one tile)
        return launch_quantize(h, n_tok * n_used, n_ff, hq, hd, n_ff / QK, s);
    }
    Q8_REQUIRE(up_gate->n_mat <= 4096, Q8_E_UNSUPPORTED, "%s: n_mat > 4096", fn);
    Q8_REQUIRE(ws != nullptr && aligned256(ws), Q8_E_WORKSPACE,
               "%s: workspace NULL or not 256-byte aligned", fn);
    Q8_REQUIRE(ws_bytes >= q8_moe_workspace_size(n_tok, n_used, up_gate->n_mat), Q8_E_WORKSPACE,
               "%s: workspace too small", fn);
    const int64_t P = n_tok * n_used;
    if (group) {
        st = launch_group(ids, n_tok, n_used, up_gate->n_mat, kTcMinPairs, (int32_t *)ws, s);
        if (st != Q8_OK) return st;
    }
    const GroupLayout L = group_layout(P, up_gate->n_mat);
    p.ws = (const int32_t *)ws;
    p.lay_count = L.count;
    p.lay_offset = L.offset;
    p.lay_list = L.list_small;
    p.lay_big = L.list_big;
    p.lay_pairs = L.pairs;
    // experts with at least kTcMinPairs rows go to the tensor cores when the
    // shape allows it; otherwise the dp4a kernel takes them too
    // (the g/u debug taps come from the dp4a kernel only)
    const bool tc = tc_eligible(up_gate, true) && P >= kTcMinPairs && !g_out && !u_out;
    p.include_big = tc ? 0 : 1;
    st = launch_up_gate(p, routed_rows(n_tok, n_used, up_gate->n_mat),
                        std::min<int64_t>(up_gate->n_mat, P), s);
    if (st != Q8_OK) return st;
    if (tc) {
        st = launch_tc(up_gate, true, xq, xd, nullptr, 0, n_tok, n_used, h, (const int32_t *)ws, s);
        if (st != Q8_OK) return st;
    }
    if (hq == nullptr) return Q8_OK;
    return launch_quantize(h, P, n_ff, hq, hd, n_ff / QK, s);
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
// Per device: the scratch address and the unique id of the context it was
// looked up in.  The address belongs to the module loaded in that context;
// when the device's context is recreated (cudaDeviceReset, a new primary
// context) the module is loaded again, possibly elsewhere, so a changed
// context id means the address is looked up again.
struct NoallocAddr {
    unsigned long long ctx_id;
    void *addr;
};
static NoallocAddr g_noalloc_addr[kMaxDevices] = {};

// The unique id of the calling thread's current context (0: none or unknown),
// through the driver entry points the runtime exposes (no link-time libcuda).
typedef int (*CtxGetCurrentFn)(void **);
typedef int (*CtxGetIdFn)(void *, unsigned long long *);
static unsigned long long current_context_id() {
    static CtxGetCurrentFn get_current = nullptr;
    static CtxGetIdFn get_id = nullptr;
    static bool resolved = false;
    if (!resolved) {
        void *f1 = nullptr, *f2 = nullptr;
        cudaDriverEntryPointQueryResult q1{}, q2{};
        if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &f1, cudaEnableDefault, &q1) ==
                cudaSuccess &&
            q1 == cudaDriverEntryPointSuccess &&
            cudaGetDriverEntryPoint("cuCtxGetId", &f2, cudaEnableDefault, &q2) == cudaSuccess &&
            q2 == cudaDriverEntryPointSuccess) {
            get_current = (CtxGetCurrentFn)f1;
            get_id = (CtxGetIdFn)f2;
        }
        resolved = true;
    }
    if (!get_current || !get_id) return 0;
    void *ctx = nullptr;
    unsigned long long id = 0;
    if (get_current(&ctx) != 0 || ctx == nullptr) return 0;
    if (get_id(ctx, &id) != 0) return 0;
    return id;
}

static q8_status noalloc_scratch_address(void **out) {
    int dev = -1;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess)
        Q8_FAIL(Q8_E_CUDA, "q8_moe_up_gate_swiglu_noalloc: cudaGetDevice: %s",
                cudaGetErrorString(e));
    Q8_REQUIRE(dev >= 0 && dev < kMaxDevices, Q8_E_UNSUPPORTED,
               "q8_moe_up_gate_swiglu_noalloc: device %d beyond %d", dev, kMaxDevices);
    std::lock_guard<std::mutex> lock(g_noalloc_mu);
    unsigned long long ctx = current_context_id();
    NoallocAddr &a = g_noalloc_addr[dev];
    if (ctx == 0 || a.addr == nullptr || a.ctx_id != ctx) {
        // set-up: the device address of the scratch in this device's current
        // context (the lookup also makes the primary context current)
        void *p = nullptr;
        e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
        if (e != cudaSuccess || p == nullptr)
            Q8_FAIL(Q8_E_CUDA, "q8_moe_up_gate_swiglu_noalloc: cudaGetSymbolAddress: %s",
                    cudaGetErrorString(e));
        if (ctx == 0) ctx = current_context_id();
        a.addr = p;
        a.ctx_id = ctx;  // 0 (id unknown): looked up again on every call
    }
    *out = a.addr;
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
    return launch_group(ids, n_tok, n_used, n_mat, kTcMinPairs, (int32_t *)ws, (cudaStream_t)stream);
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

q8_status q8_moe_up_gate_swiglu_fp32(const q8_tensor *up_gate, const float *x, int64_t n_tok,
                                     const int32_t *ids, int32_t n_used, float *h,
                                     int32_t *err_word, void *stream) {
    const char *fn = "q8_moe_up_gate_swiglu_fp32";
    q8_status st = check_tensor(up_gate, fn, false);
    if (st != Q8_OK) return st;
    Q8_REQUIRE(x && h, Q8_E_NULL, "%s: NULL pointer", fn);
    Q8_REQUIRE(up_gate->rows % 64 == 0, Q8_E_SHAPE,
               "%s: rows=%lld must be 2*n_ff with n_ff %% 32 == 0", fn, (long long)up_gate->rows);
    Q8_REQUIRE(n_tok >= 1 && n_used >= 1 && n_used <= Q8_MAX_USED, Q8_E_SHAPE,
               "%s: n_tok=%lld n_used=%d", fn, (long long)n_tok, n_used);
    Q8_REQUIRE(aligned16(x), Q8_E_ALIGN, "%s: x must be 16-byte aligned", fn);
    Q8_REQUIRE(((uintptr_t)ids & 3u) == 0 && ((uintptr_t)err_word & 3u) == 0, Q8_E_ALIGN,
               "%s: ids/err_word misaligned", fn);
    Q8_REQUIRE(n_tok * n_used <= kCtaGroupMaxPairs && up_gate->n_mat <= kCtaGroupMaxMats,
               Q8_E_UNSUPPORTED, "%s: batch of %lld pairs over %lld matrices is above the "
               "small-batch limits (%lld, %lld)", fn, (long long)(n_tok * n_used),
               (long long)up_gate->n_mat, (long long)kCtaGroupMaxPairs,
               (long long)kCtaGroupMaxMats);
    const int64_t n_ff = up_gate->rows / 2;
    UpGateParams p{};
    p.wq = up_gate->qs;
    p.wd = up_gate->d;
    p.ld_d = up_gate->ld_d;
    p.mat_stride = up_gate->mat_stride;
    p.k = (int)up_gate->k;
    p.n_ff = (int)n_ff;
    p.xf = x;
    p.h = h;
    p.n_used = n_used;
    cudaStream_t s = (cudaStream_t)stream;
    if (ids == nullptr) {
        Q8_REQUIRE(up_gate->n_mat == 1 && n_used == 1, Q8_E_SHAPE,
                   "%s: dense call (ids NULL) needs n_mat == 1, n_used == 1", fn);
        p.n_dense = (int)n_tok;
        if (n_tok >= kTcMinDense && n_tok <= kTcMaxDense && tc_eligible(up_gate, true) &&
            aligned16(x))
            return launch_tc(up_gate, true, nullptr, nullptr, x, 1, n_tok, 1, h, nullptr, s);
        return launch_up_gate(p, dense_rows(n_tok), 1, s);
    }
    const GroupLayout L = group_layout(n_tok * n_used, up_gate->n_mat);
    p.lay_count = L.count;
    p.lay_offset = L.offset;
    p.lay_list = L.list_small;
    p.lay_big = L.list_big;
    p.lay_pairs = L.pairs;
    p.include_big = 0;
    p.ids = ids;
    p.n_tok = (int)n_tok;
    p.n_mat = (int)up_gate->n_mat;
    p.err_out = err_word;
    return launch_up_gate(p, routed_rows(n_tok, n_used, up_gate->n_mat),
                          std::min<int64_t>(up_gate->n_mat, n_tok * n_used), s);
}

q8_status q8_mul_mat_id_fp32(const q8_tensor *W, const float *a, int32_t a_per_slot,
                             int64_t n_tok, const int32_t *ids, int32_t n_used, float *y,
                             int32_t *err_word, void *stream) {
    const char *fn = "q8_mul_mat_id_fp32";
    q8_status st = check_tensor(W, fn, false);
    if (st != Q8_OK) return st;
    Q8_REQUIRE(a && ids && y, Q8_E_NULL, "%s: NULL pointer", fn);
    Q8_REQUIRE(n_tok >= 1 && n_used >= 1 && n_used <= Q8_MAX_USED, Q8_E_SHAPE,
               "%s: n_tok=%lld n_used=%d", fn, (long long)n_tok, n_used);
    Q8_REQUIRE(W->rows < (1LL << 31), Q8_E_SHAPE, "%s: rows too large", fn);
    Q8_REQUIRE(aligned16(a) && ((uintptr_t)y & 3u) == 0 && ((uintptr_t)ids & 3u) == 0 &&
                   ((uintptr_t)err_word & 3u) == 0,
               Q8_E_ALIGN, "%s: a must be 16-byte aligned; y/ids/err_word 4-byte", fn);
    Q8_REQUIRE(n_tok * n_used <= kCtaGroupMaxPairs && W->n_mat <= kCtaGroupMaxMats,
               Q8_E_UNSUPPORTED, "%s: batch above the small-batch limits", fn);
    return launch_matmul_routed_ids(W, nullptr, nullptr, a, a_per_slot, n_tok, n_used, ids, y,
                                    err_word, (cudaStream_t)stream);
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
    // the fp32 calls with the grouping built in every CTA serve dense batches
    // and routed batches of at most kLayerMaxPairs pairs (one fused kernel
    // when the shapes allow); larger routed batches group once and send the
    // experts with at least kTcMinPairs rows to the tensor cores (at 16 to
    // 128 tokens of the 128-expert layer: 1.1x to 2.2x faster than the fp32
    // calls, whose dp4a kernels take every expert)
    const int64_t P = n_tok * n_used;
    const bool small = P <= kCtaGroupMaxPairs && up_gate->n_mat <= kCtaGroupMaxMats &&
                       (!routed || P <= kLayerMaxPairs);
    Q8_REQUIRE(ws != nullptr && aligned256(ws), Q8_E_WORKSPACE,
               "q8_moe_ffn: workspace NULL or not 256-byte aligned");
    Q8_REQUIRE(ws_bytes >= F.total, Q8_E_WORKSPACE, "q8_moe_ffn: workspace too small");
    cudaStream_t s = (cudaStream_t)stream;
    unsigned char *w8 = (unsigned char *)ws;
    int8_t *xq = (int8_t *)(w8 + F.xq);
    uint16_t *xd = (uint16_t *)(w8 + F.xd);
    float *h = (float *)(w8 + F.h);
    if (small) {
        // Three launches: up/gate (x quantized as it is staged; routed: the
        // grouping built in each CTA from ids), down (h quantized as it is
        // staged; dense h rows longer than the raw slot: quantized once
        // before it), combine (routed).
        int32_t *err = routed ? (int32_t *)(w8 + F.group) : nullptr;
        if (routed && layer_eligible(up_gate, down, n_tok, n_used))
            return launch_layer(up_gate, down, x, n_tok, ids, route_w, n_used, out, h,
                                (unsigned *)(w8 + F.group) + WS_BAR, err, s);
        st = q8_moe_up_gate_swiglu_fp32(up_gate, x, n_tok, ids, n_used, h, err, s);
        if (st != Q8_OK) return st;
        if (!routed) {
            if (4 * n_ff <= kRawSlotBytes)
                return launch_matmul_dense(down, nullptr, nullptr, h, n_tok, out, s);
            // h rows too long for the raw slot: every CTA of the down kernel
            // would quantize all of h from global memory (a 14336-long row:
            // about 7 us of each launch), so h is quantized once here
            int8_t *hq = (int8_t *)(w8 + F.hq);
            uint16_t *hd = (uint16_t *)(w8 + F.hd);
            st = q8_quantize_row(h, n_tok, n_ff, hq, hd, s);
            if (st != Q8_OK) return st;
            return launch_matmul_dense(down, hq, hd, nullptr, n_tok, out, s);
        }
        float *y = (float *)(w8 + F.y);
        st = q8_mul_mat_id_fp32(down, h, 1, n_tok, ids, n_used, y, nullptr, s);
        if (st != Q8_OK) return st;
        return launch_combine(y, route_w, n_tok, n_used, n_embd, out, s);
    }
    st = q8_quantize_row(x, n_tok, n_embd, xq, xd, s);
    if (st != Q8_OK) return st;
    if (!routed) {
        st = q8_moe_up_gate_swiglu(up_gate, xq, xd, n_tok, nullptr, 1, h, nullptr, nullptr,
                                   nullptr, nullptr, nullptr, 0, s);
        if (st != Q8_OK) return st;
        // the down projection quantizes h to Q8_0 as it stages it
        return launch_matmul_dense(down, nullptr, nullptr, h, n_tok, out, s);
    }
    int32_t *wsg = (int32_t *)(w8 + F.group);
    const size_t gbytes = group_bytes(n_tok * n_used, up_gate->n_mat);
    int8_t *hq = (int8_t *)(w8 + F.hq);
    uint16_t *hd = (uint16_t *)(w8 + F.hd);
    // one grouping serves the gate/up and the down projection; h is
    // quantized once, after the up/gate step, for both down kernels
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

q8_status q8_reset_errors(void) {
    if (clear_wait_errors_matmul() != Q8_OK || clear_wait_errors_moe() != Q8_OK ||
        clear_wait_errors_tc() != Q8_OK || clear_wait_errors_layer() != Q8_OK)
        Q8_FAIL(Q8_E_CUDA, "q8_reset_errors: clearing the kernels' wait flags failed");
    return Q8_OK;
}

q8_status q8_check(const void *ws, void *stream) {
    cudaStream_t s = (cudaStream_t)stream;
    int32_t flags = 0;
    cudaError_t e = cudaSuccess;
    if (ws) e = cudaMemcpyAsync(&flags, ws, sizeof flags, cudaMemcpyDeviceToHost, s);
    if (e == cudaSuccess) e = cudaStreamSynchronize(s);
    if (e != cudaSuccess) Q8_FAIL(Q8_E_CUDA, "q8_check: %s", cudaGetErrorString(e));
    int w1 = 0, w2 = 0, w3 = 0, w4 = 0;
    if (read_wait_errors_matmul(&w1) != Q8_OK || read_wait_errors_moe(&w2) != Q8_OK ||
        read_wait_errors_tc(&w3) != Q8_OK || read_wait_errors_layer(&w4) != Q8_OK)
        Q8_FAIL(Q8_E_CUDA, "q8_check: reading the kernels' wait flags failed");
    if (w1 | w2 | w3 | w4)
        Q8_FAIL(Q8_E_CUDA, "q8_check: a kernel gave up waiting for a shared-memory stage");
    if (flags & ERR_ID_RANGE) Q8_FAIL(Q8_E_BAD_ID, "q8_check: a routing id is out of range");
    if (flags & ERR_ID_REPEAT)
        Q8_FAIL(Q8_E_BAD_ID, "q8_check: a routing id repeats within a token");
    return Q8_OK;
}

}  // extern "C"
