// q8_matmul.cu -- Q8_0 x Q8_0 matrix-vector kernels: the batch-1 GEMV
// (q8_gemv), many independent GEMVs in one launch (q8_gemv_batched) and the
// matmul indexed by expert id (q8_mul_mat_id), plus the block-dot test hook.
//
// The Q8_0 decode matvec is the hot loop of the Llama 2 110M int8 decode in
// the "narray-llm" README (section "Llama 2 110M を int8 (Q8_0) で");
// mul_mat_id is ggml_mul_mat_id of the news.hada.io article on Gemma 4
// 26B-A4B Q8_0 (section 「3段階で構成された修正」), applied per routed expert.
// All of them run on the streaming engine of q8_stream.cuh.
#include <algorithm>
#include <vector>

#include "q8_internal.h"
#include "q8_stream.cuh"

namespace q8 {

// Wait timeouts of the kernels in this file (read by q8_check).
static __device__ int g_err_matmul;

q8_status read_wait_errors_matmul(int *flags) {
    cudaError_t e = cudaMemcpyFromSymbol(flags, g_err_matmul, sizeof(int));
    return e == cudaSuccess ? Q8_OK : Q8_E_CUDA;
}

q8_status clear_wait_errors_matmul() {
    const int zero = 0;
    cudaError_t e = cudaMemcpyToSymbol(g_err_matmul, &zero, sizeof(int));
    return e == cudaSuccess ? Q8_OK : Q8_E_CUDA;
}

// Consumer side of a dense Q8_0 activation set that the producer copied with
// the CTA's first tile (q8_copy_job): the quants straight into the stage,
// the fp16 scales into the upper half of the fp32 scale area, widened here
// in place.  Chunks of 2 * kCT scales: every thread reads its two, a
// barrier, then writes them; a write of scale i overwrites fp16 scales
// 2i - nd and 2i - nd + 1, which are below the chunk's end and so already
// read (all nd of them when the chunk is the last).
__device__ __forceinline__ void stage_q8_landed(const XStage &xs, int k, int n, const Ring &R,
                                                int *err) {
    mbar_wait(R.xfull, 0, err);
    const int nd = n * (k / QK);
    const uint16_t *h16 = reinterpret_cast<const uint16_t *>(xs.dx) + nd;
    const int tid = (int)threadIdx.x;
    for (int base = 0; base < nd; base += 2 * kCT) {  // the same trip count in every thread
        const int i0 = base + tid, i1 = base + kCT + tid;
        const uint16_t a = i0 < nd ? h16[i0] : (uint16_t)0;
        const uint16_t b = i1 < nd ? h16[i1] : (uint16_t)0;
        named_bar_sync(kBarConsumers, kCT);
        if (i0 < nd) xs.dx[i0] = scale_value(a);
        if (i1 < nd) xs.dx[i1] = scale_value(b);
    }
}

// Producer side: n dense Q8_0 rows (quants aq, scales ad, both contiguous
// and 16-byte aligned, n * k / 16 and n * (k / 32) / 8 whole) in two bulk
// copies on R.xfull.
__device__ __forceinline__ void q8_copy_job(const Ring &R, const Plan &pl, const int8_t *aq,
                                            const uint16_t *ad, int k, int n) {
    const uint32_t qbytes = (uint32_t)n * (uint32_t)k;
    const uint32_t dbytes = (uint32_t)n * (uint32_t)(k / QK) * 2u;
    unsigned char *base = reinterpret_cast<unsigned char *>(R.xfull) - pl.off_xfull;
    mbar_arrive_expect_tx(R.xfull, qbytes + dbytes);
    bulk_g2s_keep(base + pl.off_xq, aq, qbytes, R.xfull);
    bulk_g2s_keep(base + pl.off_xd + dbytes, ad, dbytes, R.xfull);
}

// ---------------------------------------------------------------------------
// matmul over the activation rows of each matrix.
//   dense  (ws == nullptr): matrix 0; activation rows 0..n_dense-1; output
//          row = activation row.
//   routed (ws != nullptr): the experts of the grouping list; for expert e the
//          pairs p of its list; activation row = p (a_per_slot) or p / n_used;
//          output row = p.
// Activations are Q8_0 (aq, ad) or fp32 (af, quantized while staged).
// Output y[out_row * rows + r].
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
    const float *af;
    float *y;
    const int32_t *ws;
    int64_t lay_count, lay_offset, lay_list, lay_pairs, lay_big;
    int include_big;  // the dp4a kernel also takes the tensor-core list
    int n_dense;
    int a_per_slot;
    int n_used;
    // routed with the grouping built in each CTA from ids (ws unused)
    const int32_t *ids;
    int n_tok;
    int n_mat;
    int32_t *err_out;
    // dense Q8_0 activations that the producer copies into the stage with
    // the first tile (all rows in one group, contiguous, 16-byte aligned)
    int q8_copy;
    Plan plan;
};

// Dense: an instantiation for dense calls (no grouping table, no ids), whose
// activation staging takes the wide forms (stage_q8, stage_f32).
template <int NT, bool Dense>
__global__ void __launch_bounds__(kThreadsStream, ctas_per_sm(NT))
    stream_matmul_kernel(const __grid_constant__ MatmulParams p) {
    extern __shared__ __align__(128) unsigned char smem[];
    Q8_TRACE(0);
    const Ring R = ring_init(smem, p.plan);
    Q8_TRACE(1);
    const Geo g = geo_for_k(p.k, NT);
    const int tpm = (p.rows + g.nr - 1) / g.nr;
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
                const int r0 = ti * g.nr;
                const int64_t row = (int64_t)e * p.mat_stride + r0;
                ts.q0 = p.wq + row * p.k;
                ts.d0 = p.wd + row * p.ld_d;
                ts.rows0 = min(g.nr, p.rows - r0);
                ts.k = p.k;
                ts.ld_d = (int)p.ld_d;
                return ts;
            };
            if (p.af && R.raw_rows > 0) {
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
                            const int r = (!routed || p.a_per_slot) ? pr : pr / p.n_used;
                            return p.af + (int64_t)r * p.k;
                        }, &g_err_matmul);
                    }
                };
                produce(R, tb, te, src, &g_err_matmul, jobs, !routed);
            } else if constexpr (Dense) {
                if (p.q8_copy) {
                    // the rows may come from the preceding grid: the first
                    // tile goes out before the wait, the rows right after
                    // it, ahead of the rest of the stream
                    bool copied = false;
                    auto qjob = [&](int64_t, int when) {
                        if (when != 0 || copied) return;
                        q8_copy_job(R, p.plan, p.aq, p.ad, p.k, p.n_dense);
                        copied = true;
                    };
                    produce(R, tb, te, src, &g_err_matmul, qjob, true);
                } else {
                    produce(R, tb, te, src, &g_err_matmul);
                }
            } else {
                produce(R, tb, te, src, &g_err_matmul);
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
        mbar_wait(&R.full[s], (it / R.stages) & 1, &g_err_matmul);
        Q8_TRACE(6);
        const int mi = (int)(t / tpm), ti = (int)(t % tpm);
        const int e = routed ? expert(mi) : 0;
        const int cnt = routed ? tab[p.lay_count + e] : p.n_dense;
        const int32_t *plist = routed ? tab + p.lay_pairs + tab[p.lay_offset + e] : nullptr;
        const int r0 = ti * g.nr;
        const int rows_valid = min(g.nr, p.rows - r0);
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
                    return (!routed || p.a_per_slot) ? pr : pr / p.n_used;
                };
                if (p.af) {
                    stage_job_f32<Dense>(R, J, xs, p.af, p.k, nx, arow, &g_err_matmul);
                } else if constexpr (Dense) {
                    if (p.q8_copy)
                        stage_q8_landed(xs, p.k, nx, R, &g_err_matmul);
                    else
                        stage_q8<Dense>(xs, p.aq, p.ad, p.k, nx, arow);
                } else {
                    stage_q8<Dense>(xs, p.aq, p.ad, p.k, nx, arow);
                }
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
                        // whole rows per warp: each sum is final, written
                        // by the lane that holds it (no barrier)
                        warp_rows<NTC>(R.qs(s), R.d(s), p.k, (int)p.ld_d, g, xs, tg, n,
                                       [&](int row, int tt, float v) {
                                           if (row < rows_valid && tt < n) {
                                               const int pr = plist ? plist[x0 + tg + tt]
                                                                    : x0 + tg + tt;
                                               p.y[(int64_t)pr * p.rows + r0 + row] = v;
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
                    if (grp == n_grp - 1 && tg + NT >= nx) {  // last read of this stage
                        __syncwarp();
                        if ((threadIdx.x & 31) == 0) mbar_arrive(&R.empty[s]);
                    }
                    named_bar_sync(kBarConsumers, kCT);
                    Q8_TRACE(9);
                    for (int i = threadIdx.x; i < rows_valid * n; i += kCT) {
                        const int row = i / n;
                        const int tt = i - row * n;
                        const int pr = plist ? plist[x0 + tg + tt] : x0 + tg + tt;
                        p.y[(int64_t)pr * p.rows + r0 + row] = part_sum<NTC>(part, g, row, tt);
                    }
                    Q8_TRACE(10);
                });
                buf ^= 1;
            }
        }
    }
}

static int g_num_sms[64];

int num_sms() {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 148;
    if (g_num_sms[dev] == 0) {
        int n = 0;
        if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0)
            n = 148;
        g_num_sms[dev] = n;
    }
    return g_num_sms[dev];
}

// rp: rows per compute pass (the kernel's NT) and rows staged at once;
// max_tiles: an upper bound of the tile count (sizes the grid).
q8_status launch_matmul(const MatmulParams &base, RowPlan rp, int64_t max_tiles,
                        cudaStream_t s) {
    MatmulParams p = base;
    const int nt = pick_nt(rp.nt_rows);
    const int tab_words =
        p.ids ? (int)group_layout((int64_t)p.n_tok * p.n_used, p.n_mat).words : 0;
    int tq, td;
    tile_bytes(geo_for_k(p.k, nt), p.k, p.ld_d, &tq, &td);
    if (!make_plan(tq, td, p.k, (int)std::min<int64_t>(rp.x_rows, kMaxXRows), nt, &p.plan,
                   tab_words, p.af != nullptr && aligned16(p.af)))
        Q8_FAIL(Q8_E_UNSUPPORTED, "matmul: k=%d does not fit the shared-memory plan", p.k);
    const int grid = (int)std::max<int64_t>(1, std::min<int64_t>((int64_t)num_sms() * p.plan.ctas, max_tiles));
    const int64_t nd = (int64_t)p.n_dense * (p.k / QK);
    p.q8_copy = !p.ids && !p.ws && p.aq && p.ad && aligned16(p.aq) && aligned16(p.ad) &&
                p.n_dense >= 1 && p.n_dense <= p.plan.xmax && p.k <= p.plan.max_nb * QK &&
                nd % 8 == 0;
    if (!p.ids && !p.ws) {
        switch (nt) {
            case 1: return launch_stream(stream_matmul_kernel<1, true>, grid, p.plan.bytes, s, p, "matmul");
            case 2: return launch_stream(stream_matmul_kernel<2, true>, grid, p.plan.bytes, s, p, "matmul");
            case 4: return launch_stream(stream_matmul_kernel<4, true>, grid, p.plan.bytes, s, p, "matmul");
            default: return launch_stream(stream_matmul_kernel<8, true>, grid, p.plan.bytes, s, p, "matmul");
        }
    }
    switch (nt) {
        case 1: return launch_stream(stream_matmul_kernel<1, false>, grid, p.plan.bytes, s, p, "matmul");
        case 2: return launch_stream(stream_matmul_kernel<2, false>, grid, p.plan.bytes, s, p, "matmul");
        case 4: return launch_stream(stream_matmul_kernel<4, false>, grid, p.plan.bytes, s, p, "matmul");
        default: return launch_stream(stream_matmul_kernel<8, false>, grid, p.plan.bytes, s, p, "matmul");
    }
}

// mul_mat_id over grouping tables already written to ws.  af: fp32
// activations instead of aq/ad (quantized while staged).
q8_status launch_matmul_routed(const q8_tensor *W, const int8_t *aq, const uint16_t *ad,
                               const float *af, int a_per_slot, int64_t n_tok, int32_t n_used,
                               float *y, const int32_t *ws, cudaStream_t s) {
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
    p.af = af;
    p.y = y;
    p.ws = ws;
    p.lay_count = L.count;
    p.lay_offset = L.offset;
    p.lay_list = L.list_small;
    p.lay_big = L.list_big;
    p.lay_pairs = L.pairs;
    p.include_big = 0;
    p.a_per_slot = a_per_slot ? 1 : 0;
    p.n_used = n_used;
    // experts with at least kTcMinPairs rows go to the tensor cores when the
    // shape allows it; otherwise the dp4a kernel takes them too
    const bool tc = tc_eligible(W, false) && P >= kTcMinPairs;
    p.include_big = tc ? 0 : 1;
    const Geo g = geo_for_k(p.k, 8);
    const int64_t tiles = std::min<int64_t>(W->n_mat, P) * ((p.rows + g.nr - 1) / g.nr);
    q8_status st = launch_matmul(p, routed_rows(n_tok, n_used, W->n_mat), tiles, s);
    if (st != Q8_OK || !tc) return st;
    return launch_tc(W, false, aq, ad, af, a_per_slot, n_tok, n_used, y, ws, s);
}

// mul_mat_id with the grouping built in each CTA from ids (small batches);
// routing-id errors go to *err_out.
q8_status launch_matmul_routed_ids(const q8_tensor *W, const int8_t *aq, const uint16_t *ad,
                                   const float *af, int a_per_slot, int64_t n_tok,
                                   int32_t n_used, const int32_t *ids, float *y,
                                   int32_t *err_out, cudaStream_t s) {
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
    p.af = af;
    p.y = y;
    p.ws = nullptr;
    p.lay_count = L.count;
    p.lay_offset = L.offset;
    p.lay_list = L.list_small;
    p.lay_big = L.list_big;
    p.lay_pairs = L.pairs;
    p.include_big = 0;
    p.a_per_slot = a_per_slot ? 1 : 0;
    p.n_used = n_used;
    p.ids = ids;
    p.n_tok = (int)n_tok;
    p.n_mat = (int)W->n_mat;
    p.err_out = err_out;
    const Geo g = geo_for_k(p.k, 8);
    const int64_t tiles = std::min<int64_t>(W->n_mat, P) * ((p.rows + g.nr - 1) / g.nr);
    return launch_matmul(p, routed_rows(n_tok, n_used, W->n_mat), tiles, s);
}

// Dense matmul of fp32 (af) or Q8_0 (aq/ad) activation rows: y = W a.
q8_status launch_matmul_dense(const q8_tensor *W, const int8_t *aq, const uint16_t *ad,
                              const float *af, int64_t n_tok, float *y, cudaStream_t s) {
    // a real (small) dense contraction: the tensor cores, one pass over W
    if (n_tok >= kTcMinDense && n_tok <= kTcMaxDense && tc_eligible(W, false) &&
        (af == nullptr || aligned16(af)))
        return launch_tc(W, false, aq, ad, af, 1, n_tok, 1, y, nullptr, s);
    const Geo g = geo_for_k((int)W->k, 8);
    const int64_t tiles = (W->rows + g.nr - 1) / g.nr;
    for (int64_t t0 = 0; t0 < n_tok; t0 += kMaxXRows) {
        const int64_t nt = std::min<int64_t>(kMaxXRows, n_tok - t0);
        MatmulParams p{};
        p.wq = W->qs;
        p.wd = W->d;
        p.ld_d = W->ld_d;
        p.mat_stride = W->mat_stride;
        p.k = (int)W->k;
        p.rows = (int)W->rows;
        p.aq = aq ? aq + t0 * W->k : nullptr;
        p.ad = ad ? ad + t0 * (W->k / QK) : nullptr;
        p.af = af ? af + t0 * W->k : nullptr;
        p.y = y + t0 * W->rows;
        p.ws = nullptr;
        p.n_dense = (int)nt;
        q8_status st = launch_matmul(p, dense_rows(nt), tiles, s);
        if (st != Q8_OK) return st;
    }
    return Q8_OK;
}

// ---------------------------------------------------------------------------
// Batched GEMV: independent problems, fp32 inputs quantized while staged.
// ---------------------------------------------------------------------------
struct GemvProblem {
    const int8_t *wq;
    const uint16_t *wd;
    const float *x;
    float *y;
    int ld_d;
    int k;
    int rows;
    int tile_begin;
};

constexpr int kGemvMaxGrid = 1024;

struct GemvBatchParams {
    int n_desc;
    int n_tok;
    int total_tiles;
    int grid;
    Plan plan;
    GemvProblem pr[Q8_MAX_GEMV_DESC];
    int cta_begin[kGemvMaxGrid + 1];      // CTA b takes tiles [cta_begin[b], cta_begin[b+1])
    uint8_t first_problem[kGemvMaxGrid];  // problem of each CTA's first tile
};


// One decode row (n_tok == 1) through the tiles [t0, t1) of one problem whose
// rows a warp takes whole (k <= 4096), with RPW rows per warp and ITERS 32-block
// steps per row.  The same arithmetic, in the same order, as warp_rows (so the
// same bits): per lane, block sums scaled and added in block order, then the
// reduce-scatter tree.  What it saves is the generic path's per-tile work:
// the problem is held in registers, the lane's activation blocks are loaded
// once for the whole run, the row addresses are fixed per warp, and there is
// one tile loop with no dispatch inside.  Returns the ring position after t1.
template <int RPW, int ITERS>
__device__ __forceinline__ int gemv_run(const Ring &R, const XStage &xs, const GemvProblem &q,
                                        const Geo &g, int64_t t0, int64_t t1, int it) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int k = q.k, nb = k / QK, ld_d = q.ld_d;
    const int h0 = ((lane >> 2) & 1) * 16, h1 = 16 - h0;
    const int row0 = warp * RPW;
    uint4 xa[ITERS], xb[ITERS];
    float dx[ITERS];
#pragma unroll
    for (int i = 0; i < ITERS; ++i) {
        const int kb = i * 32 + lane;
        xa[i] = xb[i] = make_uint4(0u, 0u, 0u, 0u);
        dx[i] = 0.0f;
        if (kb < nb) {
            xa[i] = *reinterpret_cast<const uint4 *>(xs.q + kb * QK + h0);
            xb[i] = *reinterpret_cast<const uint4 *>(xs.q + kb * QK + h1);
            dx[i] = xs.dx[kb];
        }
    }
    constexpr int VP = pow2_ceil(RPW);
    const int idx = reduce_scatter_index<VP>(lane);
    const bool writer = (lane & (32 / VP - 1)) == 0 && idx < RPW;
    for (int64_t t = t0; t < t1; ++t, ++it) {
        const int s = it % R.stages;
        mbar_wait(&R.full[s], (it / R.stages) & 1, &g_err_matmul);
        Q8_TRACE(6);
        const int r0 = (int)(t - q.tile_begin) * g.nr;
        const int8_t *sq = R.qs(s) + (size_t)row0 * k;
        const uint16_t *sd = R.d(s) + (size_t)row0 * ld_d;
        float acc[RPW];
#pragma unroll
        for (int r = 0; r < RPW; ++r) acc[r] = 0.0f;
#pragma unroll
        for (int i = 0; i < ITERS; ++i) {
            const int kb = i * 32 + lane;
            if (kb < nb) {
                uint4 w0[RPW], w1[RPW];
                float dw[RPW];
#pragma unroll
                for (int r = 0; r < RPW; ++r) {
                    const int8_t *wp = sq + (size_t)r * k + kb * QK;
                    w0[r] = *reinterpret_cast<const uint4 *>(wp + h0);
                    w1[r] = *reinterpret_cast<const uint4 *>(wp + h1);
                    dw[r] = scale_value(sd[(size_t)r * ld_d + kb]);
                }
#pragma unroll
                for (int r = 0; r < RPW; ++r) {
                    const int sum = block_dot(w0[r], w1[r], xa[i], xb[i]);
                    acc[r] = fmaf(dw[r] * dx[i], small_int_to_float(sum), acc[r]);
                }
            }
        }
        float a[VP];
#pragma unroll
        for (int i = 0; i < VP; ++i) a[i] = i < RPW ? acc[i] : 0.0f;
        const float v = warp_reduce_scatter<VP>(a);
        __syncwarp();
        if (lane == 0) mbar_arrive(&R.empty[s]);
        Q8_TRACE(8);
        if (writer && row0 + idx < q.rows - r0 && row0 + idx < g.nr) q.y[r0 + row0 + idx] = v;
    }
    return it;
}

template <int NT>
__global__ void __launch_bounds__(kThreadsStream, ctas_per_sm(NT))
    gemv_batched_kernel(const __grid_constant__ GemvBatchParams p) {
    extern __shared__ __align__(128) unsigned char smem[];
    Q8_TRACE(0);
    const Ring R = ring_init(smem, p.plan);
    Q8_TRACE(1);
    griddep_launch_dependents();
    const int64_t tb = p.cta_begin[blockIdx.x], te = p.cta_begin[blockIdx.x + 1];
    if ((threadIdx.x >> 5) == kCW) {
        if ((threadIdx.x & 31) == 0 && tb < te) {
            int cur = p.first_problem[blockIdx.x];
            auto src = [&](int64_t t) {
                while (cur + 1 < p.n_desc && p.pr[cur + 1].tile_begin <= t) ++cur;
                const GemvProblem &q = p.pr[cur];
                const Geo g = geo_for_k(q.k, NT);
                const int r0 = (int)(t - q.tile_begin) * g.nr;
                TileSrc ts{};
                ts.q0 = q.wq + (int64_t)r0 * q.k;
                ts.d0 = q.wd + (int64_t)r0 * q.ld_d;
                ts.rows0 = min(g.nr, q.rows - r0);
                ts.k = q.k;
                ts.ld_d = q.ld_d;
                return ts;
            };
            if (R.raw_rows > 0) {
                XJobs J;
                int jc = cur;
                const int xmax = p.plan.xmax;
                const int n_grp = (p.n_tok + xmax - 1) / xmax;
                auto jobs = [&](int64_t t, int when) {
                    while (jc + 1 < p.n_desc && p.pr[jc + 1].tile_begin <= t) ++jc;
                    const GemvProblem &q = p.pr[jc];
                    for (int grp = when; grp < (when == 0 ? min(1, n_grp) : n_grp); ++grp) {
                        const int x0 = grp * xmax;
                        produce_job(R, J, jc, grp, min(xmax, p.n_tok - x0), q.k,
                                    [&](int j) { return q.x + (int64_t)(x0 + j) * q.k; },
                                    &g_err_matmul);
                    }
                };
                // The activation rows go first: under the weight stream of all
                // CTAs, a copy queued behind this CTA's first weight tiles lands
                // microseconds later, and no consumer can start before it.  So
                // the producer waits for the preceding grid, copies the first
                // problem's x, then streams the weights in order.
                griddep_wait();
                produce(R, tb, te, src, &g_err_matmul, jobs, false);
            } else {
                produce(R, tb, te, src, &g_err_matmul);
            }
        }
        return;
    }
    griddep_wait();
    Q8_TRACE(2);
    const XStage xs{reinterpret_cast<int8_t *>(smem + p.plan.off_xq),
                    reinterpret_cast<float *>(smem + p.plan.off_xd)};
    float *part0 = reinterpret_cast<float *>(smem + p.plan.off_part);
    const int xmax = p.plan.xmax;
    int buf = 0, staged = -1, staged_grp = -1, it = 0;
    int cur = p.first_problem[blockIdx.x];
    XJobs J;
    bool unsynced = false;  // passes without a barrier since the last one
    for (int64_t t = tb; t < te; ++t, ++it) {
        while (cur + 1 < p.n_desc && p.pr[cur + 1].tile_begin <= t) ++cur;
        if constexpr (NT == 1) {
            // one decode row, whole rows per warp: the run of this problem's
            // tiles in one tight loop (gemv_run)
            const GemvProblem qv = p.pr[cur];
            const Geo gv = geo_for_k(qv.k, 1);
            if (p.n_tok == 1 && gv.wpr == 1) {
                const int64_t t1 =
                    cur + 1 < p.n_desc ? min(te, (int64_t)p.pr[cur + 1].tile_begin) : te;
                if (cur != staged) {
                    if (unsynced) named_bar_sync(kBarConsumers, kCT);
                    stage_job_f32<true>(R, J, xs, qv.x, qv.k, 1, [](int j) { return j; },
                                  &g_err_matmul);
                    named_bar_sync(kBarConsumers, kCT);
                    Q8_TRACE(7);
                    staged = cur;
                    staged_grp = 0;
                }
                // 32-block steps per row: 1 (k <= 1024), 2 (k <= 2048) or 4
                const int iters = qv.k <= 1024 ? 1 : qv.k <= 2048 ? 2 : 4;
                if (gv.rpw == 5 && iters == 1)
                    it = gemv_run<5, 1>(R, xs, qv, gv, t, t1, it);
                else if (gv.rpw == 4 && iters == 1)
                    it = gemv_run<4, 1>(R, xs, qv, gv, t, t1, it);
                else if (gv.rpw == 3 && iters == 1)
                    it = gemv_run<3, 1>(R, xs, qv, gv, t, t1, it);
                else if (gv.rpw == 2 && iters == 1)
                    it = gemv_run<2, 1>(R, xs, qv, gv, t, t1, it);
                else if (gv.rpw == 2 && iters == 2)
                    it = gemv_run<2, 2>(R, xs, qv, gv, t, t1, it);
                else if (gv.rpw == 1 && iters == 1)
                    it = gemv_run<1, 1>(R, xs, qv, gv, t, t1, it);
                else if (gv.rpw == 1 && iters == 2)
                    it = gemv_run<1, 2>(R, xs, qv, gv, t, t1, it);
                else
                    it = gemv_run<1, 4>(R, xs, qv, gv, t, t1, it);
                unsynced = true;
                t = t1 - 1;  // the loop's increments step to t1 and keep it
                --it;
                continue;
            }
        }
        const GemvProblem &q = p.pr[cur];
        const Geo g = geo_for_k(q.k, NT);
        const int s = it % R.stages;
        mbar_wait(&R.full[s], (it / R.stages) & 1, &g_err_matmul);
        Q8_TRACE(6);
        const int r0 = (int)(t - q.tile_begin) * g.nr;
        const int rows_valid = min(g.nr, q.rows - r0);
        const int n_grp = (p.n_tok + xmax - 1) / xmax;
        for (int grp = 0; grp < n_grp; ++grp) {
            const int x0 = grp * xmax;
            const int nx = min(xmax, p.n_tok - x0);
            if (cur != staged || grp != staged_grp) {
                // after passes without a barrier every warp must be done
                // with the staged rows before they are replaced
                if (unsynced) named_bar_sync(kBarConsumers, kCT);
                unsynced = false;
                stage_job_f32<true>(R, J, xs, q.x, q.k, nx, [&](int j) { return x0 + j; },
                              &g_err_matmul);
                named_bar_sync(kBarConsumers, kCT);
                Q8_TRACE(7);
                staged = cur;
                staged_grp = grp;
            }
            for (int tg = 0; tg < nx; tg += NT) {
                const int n = min(NT, nx - tg);
                float *part = part0 + buf * kPartRows * NT;
                with_nt<NT>(n, [&](auto ntc) {
                    constexpr int NTC = decltype(ntc)::value;
                    if (g.wpr == 1) {
                        // whole rows per warp: each sum is final, written
                        // by the lane that holds it (no barrier)
                        warp_rows<NTC>(R.qs(s), R.d(s), q.k, q.ld_d, g, xs, tg, n,
                                       [&](int row, int tt, float v) {
                                           if (row < rows_valid && tt < n)
                                               q.y[(int64_t)(x0 + tg + tt) * q.rows + r0 + row] = v;
                                       });
                        Q8_TRACE(8);
                        if (grp == n_grp - 1 && tg + NT >= nx) {
                            __syncwarp();
                            if ((threadIdx.x & 31) == 0) mbar_arrive(&R.empty[s]);
                        }
                        unsynced = true;
                        return;
                    }
                    warp_rows_to_part<NTC>(R.qs(s), R.d(s), q.k, q.ld_d, g, xs, tg, n, part);
                    Q8_TRACE(8);
                    if (grp == n_grp - 1 && tg + NT >= nx) {
                        __syncwarp();
                        if ((threadIdx.x & 31) == 0) mbar_arrive(&R.empty[s]);
                    }
                    named_bar_sync(kBarConsumers, kCT);
                    Q8_TRACE(9);
                    for (int i = threadIdx.x; i < rows_valid * n; i += kCT) {
                        const int row = i / n;
                        const int tt = i - row * n;
                        q.y[(int64_t)(x0 + tg + tt) * q.rows + r0 + row] =
                            part_sum<NTC>(part, g, row, tt);
                    }
                    Q8_TRACE(10);
                });
                buf ^= 1;
            }
        }
    }
}

// ---------------------------------------------------------------------------
// Test hook: per-block int32 dots through block_dot.
// A row index outside [0, n_w_rows) writes INT32_MIN for each of its blocks
// and reads nothing.
// ---------------------------------------------------------------------------
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

}  // namespace q8

using namespace q8;

extern "C" {

q8_status q8_gemv(const q8_tensor *W, const int8_t *xq, const uint16_t *xd, int64_t n_tok,
                  float *y, void *stream) {
    q8_status st = check_tensor(W, "q8_gemv: W", true);
    if (st != Q8_OK) return st;
    Q8_REQUIRE(xq && xd && y, Q8_E_NULL, "q8_gemv: NULL pointer");
    Q8_REQUIRE(n_tok >= 1 && n_tok <= 4096, Q8_E_SHAPE, "q8_gemv: n_tok=%lld (1..4096)",
               (long long)n_tok);
    Q8_REQUIRE(W->rows < (1LL << 31), Q8_E_SHAPE, "q8_gemv: rows too large");
    Q8_REQUIRE(aligned16(xq), Q8_E_ALIGN, "q8_gemv: xq must be 16-byte aligned");
    Q8_REQUIRE(((uintptr_t)xd & 1u) == 0 && ((uintptr_t)y & 3u) == 0, Q8_E_ALIGN,
               "q8_gemv: xd/y misaligned");
    return launch_matmul_dense(W, xq, xd, nullptr, n_tok, y, (cudaStream_t)stream);
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
        st = launch_group(ids, n_tok, n_used, W->n_mat, kTcMinPairs, (int32_t *)ws, s);
        if (st != Q8_OK) return st;
    }
    return launch_matmul_routed(W, aq, ad, nullptr, a_per_slot, n_tok, n_used, y,
                                (const int32_t *)ws, s);
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
    int64_t tiles = 0;
    int max_k = 32, max_tq = 0, max_td = 0;
    const int nt = pick_nt(n_tok);
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
        q.ld_d = (int)d.W.ld_d;
        q.k = (int)d.W.k;
        q.rows = (int)d.W.rows;
        q.tile_begin = (int)tiles;
        const Geo g = geo_for_k(q.k, nt);
        tiles += (d.W.rows + g.nr - 1) / g.nr;
        max_k = std::max(max_k, q.k);
        int tq, td;
        tile_bytes(g, q.k, q.ld_d, &tq, &td);
        max_tq = std::max(max_tq, tq);
        max_td = std::max(max_td, td);
    }
    Q8_REQUIRE(tiles < (1LL << 31), Q8_E_SHAPE, "q8_gemv_batched: too many tiles");
    p.total_tiles = (int)tiles;
    if (!make_plan(max_tq, max_td, max_k, (int)std::min<int64_t>(n_tok, kMaxXRows), nt, &p.plan,
                   0, true))
        Q8_FAIL(Q8_E_UNSUPPORTED, "q8_gemv_batched: k=%d does not fit the plan", max_k);
    const int grid = (int)std::max<int64_t>(
        1, std::min<int64_t>(std::min<int64_t>((int64_t)num_sms() * p.plan.ctas, tiles),
                             kGemvMaxGrid));
    p.grid = grid;
    // Contiguous runs of tiles of equal cost: a tile costs its bytes, and the
    // first tile of a problem also the restaging of the activations that it
    // makes a CTA pay (about 0.7 of a tile's time).  Also the problem of each
    // CTA's first tile, so that no thread searches the problem list.
    {
        std::vector<double> cost((size_t)tiles);
        double total = 0.0;
        for (int i = 0; i < n_desc; ++i) {
            const GemvProblem &q = p.pr[i];
            const Geo g = geo_for_k(q.k, nt);
            const int64_t nt = (q.rows + g.nr - 1) / g.nr;
            const double tb_bytes = (double)g.nr * q.k * 1.0625;
            for (int64_t t = 0; t < nt; ++t) {
                cost[(size_t)(q.tile_begin + t)] = tb_bytes * (t == 0 ? 1.7 : 1.0);
                total += cost[(size_t)(q.tile_begin + t)];
            }
        }
        double acc = 0.0;
        int64_t t = 0;
        p.cta_begin[0] = 0;
        for (int b = 1; b < grid; ++b) {
            const double target = total * b / grid;
            while (t < tiles && acc + 0.5 * cost[(size_t)t] < target) acc += cost[(size_t)t++];
            // keep at least one tile for each remaining CTA
            const int64_t max_t = tiles - (grid - b);
            if (t > max_t) {
                while (t > max_t) acc -= cost[(size_t)--t];
            }
            if (t < p.cta_begin[b - 1] + 1) acc += cost[(size_t)t++];
            p.cta_begin[b] = (int)t;
        }
        p.cta_begin[grid] = (int)tiles;
        for (int b = 0, cur = 0; b < grid; ++b) {
            while (cur + 1 < n_desc && p.pr[cur + 1].tile_begin <= p.cta_begin[b]) ++cur;
            p.first_problem[b] = (uint8_t)cur;
        }
    }
    cudaStream_t s = (cudaStream_t)stream;
    switch (nt) {
        case 1: return launch_stream(gemv_batched_kernel<1>, grid, p.plan.bytes, s, p, "gemv_batched");
        case 2: return launch_stream(gemv_batched_kernel<2>, grid, p.plan.bytes, s, p, "gemv_batched");
        case 4: return launch_stream(gemv_batched_kernel<4>, grid, p.plan.bytes, s, p, "gemv_batched");
        default: return launch_stream(gemv_batched_kernel<8>, grid, p.plan.bytes, s, p, "gemv_batched");
    }
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
