// q8_layer.cu -- the routed MoE feed-forward step of a small batch as ONE
// persistent kernel: the expert grouping, the fused up/gate + SwiGLU, a
// grid-wide barrier, then the down projection with the routing-weight
// combine.  It is the fused form of the fallback chain the news.hada.io
// article on Gemma 4 26B-A4B describes (section 「3段階で構成された修正」:
// mul_mat_id over the gate and up slices of up_gate_exps, fused_mul_unary
// SILU, mul_mat_id over down_exps, then the weighted sum over the routed
// experts).  At one decode token a layer reads about 50 MB of weights, a few
// microseconds of HBM time, so separate launches (each with its own start-up
// and drain) dominate; here the weight stream runs through one ring from the
// first up/gate tile to the last down tile, and the down weights are already
// in flight while the grid waits for h.
//
// Grid: one CTA per SM, all co-resident (cooperative launch), each with the
// streaming engine of q8_stream.cuh (one producer warp, 8 consumer warps).
//  phase A  tiles of 8 gate rows + the 8 matching up rows of one routed
//           expert (k <= 4096: whole rows per warp); x rows are copied by the
//           producer and quantized in shared memory; h goes to global memory.
//  barrier  all CTAs' h is written (bounded wait).
//  phase B  units of kLayerNrb (8) down rows; a stage holds those rows of up to 8
//           experts (one per warp).  Every CTA stages all pairs' h as Q8_0,
//           computes y for its rows, then forms out[t] = sum_s p[t][s] y[t][s]
//           in s order for the unit's rows (the combine_kernel fma chain).
// The outputs are bit-identical to the three-launch path (same tiles' row
// sums, same h quantization, same combine order).
#include <algorithm>

#include "q8_internal.h"
#include "q8_stream.cuh"

namespace q8 {

static __device__ int g_err_layer;

q8_status read_wait_errors_layer(int *flags) {
    cudaError_t e = cudaMemcpyFromSymbol(flags, g_err_layer, sizeof(int));
    return e == cudaSuccess ? Q8_OK : Q8_E_CUDA;
}

constexpr int kLayerNrb = 8;  // down rows per unit (rows per warp in phase B)
constexpr int kLayerNT = 4;   // activation rows per pass (template bound)

struct LayerParams {
    const int8_t *ug_q;
    const uint16_t *ug_d;
    int64_t ug_ld_d, ug_stride;
    const int8_t *dn_q;
    const uint16_t *dn_d;
    int64_t dn_ld_d, dn_stride;
    int k;     // n_embd (up/gate K, down rows)
    int n_ff;  // down K
    const float *x;
    const int32_t *ids;
    const float *route_w;
    float *out;
    float *h;       // [P][n_ff] scratch
    unsigned *bar;  // grid barrier {arrivals, generation}
    int32_t *err_out;
    int n_tok, n_used, n_mat;
    int64_t lay_count, lay_offset, lay_list, lay_big, lay_pairs;
    int off_hq, off_hd, off_y, off_inv;  // phase-B areas
    Plan plan;
};

__device__ __forceinline__ unsigned ld_acquire_u32(const unsigned *p) {
    unsigned v;
    asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    return v;
}

// Barrier of all CTAs of a co-resident grid, entered by one thread per CTA
// after its CTA's global writes (ordered by a CTA barrier before the call).
// bar[0] counts arrivals and is reset to 0 by the last one, which then
// advances the generation bar[1]; the others wait for the generation to move.
// Bounded: after kWaitLimitNs the wait records Q8_WAIT_TIMEOUT and returns
// false (the barrier word is then left inconsistent: q8_check reports it).
__device__ __forceinline__ bool grid_barrier(unsigned *bar, unsigned n, int *err) {
    const unsigned gen = ld_acquire_u32(bar + 1);
    __threadfence();
    const unsigned old = atomicAdd(bar, 1u);
    if (old == n - 1) {
        atomicExch(bar, 0u);
        __threadfence();
        atomicAdd(bar + 1, 1u);
        return true;
    }
    const uint64_t t0 = globaltimer_ns();
    while (ld_acquire_u32(bar + 1) == gen) {
        if (globaltimer_ns() - t0 > kWaitLimitNs) {
            atomicOr(err, Q8_WAIT_TIMEOUT);
            return false;
        }
        __nanosleep(64);
    }
    __threadfence();
    return true;
}

// Quantize fp32 rows written in this launch by other CTAs (so loaded at L2,
// not through L1): n rows of k floats, row j at src + arow(j) * k, into the
// stage, one thread per 32-block.
template <class RowFn>
__device__ __forceinline__ void stage_f32_l2(const XStage &xs, const float *src, int k, int n,
                                             RowFn arow) {
    const int nb = k / QK;
    for (int blk = threadIdx.x; blk < n * nb; blk += kCT) {
        const int j = blk / nb;
        const int b = blk - j * nb;
        const float4 *p = reinterpret_cast<const float4 *>(src + (int64_t)arow(j) * k + b * QK);
        float v[32];
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            const float4 f = __ldcg(p + i);
            v[4 * i] = f.x;
            v[4 * i + 1] = f.y;
            v[4 * i + 2] = f.z;
            v[4 * i + 3] = f.w;
        }
        uint32_t q[8];
        const float d32 = quantize_block_thread(v, q);
        uint4 *dst = reinterpret_cast<uint4 *>(xs.q + (size_t)j * k + b * QK);
        dst[0] = make_uint4(q[0], q[1], q[2], q[3]);
        dst[1] = make_uint4(q[4], q[5], q[6], q[7]);
        xs.dx[(size_t)j * nb + b] = scale_value(scale_bits(d32));
    }
}

template <int NT>
__global__ void __launch_bounds__(kThreadsStream, 1) moe_layer_kernel(const __grid_constant__ LayerParams p) {
    extern __shared__ __align__(128) unsigned char smem[];
    Q8_TRACE(0);
    const Ring R = ring_init(smem, p.plan);
    Q8_TRACE(1);
    griddep_wait();  // x, ids and route_w may come from the preceding kernel
    griddep_launch_dependents();
    int32_t *tab = reinterpret_cast<int32_t *>(smem + p.plan.off_tab);
    {
        GroupLayout L{};
        L.count = p.lay_count;
        L.offset = p.lay_offset;
        L.list_small = p.lay_list;
        L.list_big = p.lay_big;
        L.pairs = p.lay_pairs;
        cta_group(p.ids, p.n_tok, p.n_used, p.n_mat, L, tab, p.err_out);
    }
    Q8_TRACE(3);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int n_exp = tab[WS_N_SMALL];
    const Geo ga = geo_pair_for_k(p.k);
    const int half = ga.nr / 2;
    const int tpm = p.n_ff / half;
    const int units = (p.k + kLayerNrb - 1) / kLayerNrb;
    const int sg_per_unit = (n_exp + kCW - 1) / kCW;
    const int xmax = p.plan.xmax;
    int64_t ta0, ta1, ub0, ub1;
    my_tiles((int64_t)n_exp * tpm, &ta0, &ta1);
    my_tiles(units, &ub0, &ub1);
    auto expert = [&](int i) { return tab[p.lay_list + i]; };

    if (warp == kCW) {  // ---------------- producer
        if (lane == 0) {
            int it = 0;
            XJobs J;
            auto jobs = [&](int64_t t, int when) {
                const int e = expert((int)(t / tpm));
                const int cnt = tab[p.lay_count + e];
                const int32_t *plist = tab + p.lay_pairs + tab[p.lay_offset + e];
                const int n_grp = (cnt + xmax - 1) / xmax;
                for (int grp = when; grp < (when == 0 ? min(1, n_grp) : n_grp); ++grp) {
                    const int x0 = grp * xmax;
                    produce_job(R, J, (int)(t / tpm), grp, min(xmax, cnt - x0), p.k, [&](int j) {
                        return p.x + (int64_t)(plist[x0 + j] / p.n_used) * p.k;
                    }, &g_err_layer);
                }
            };
            for (int64_t t = ta0; t < ta1; ++t, ++it) {  // phase A: gate/up tiles
                const int s = it % R.stages;
                if (R.raw_rows > 0) jobs(t, 0);
                if (it >= R.stages) mbar_wait(&R.empty[s], (it / R.stages - 1) & 1, &g_err_layer);
                const int e = expert((int)(t / tpm));
                const int ti = (int)(t % tpm);
                const int64_t grow = (int64_t)e * p.ug_stride + (int64_t)ti * half;
                const int64_t urow = grow + p.n_ff;
                Q8_TRACE(21);
                const uint32_t qb = (uint32_t)(half * p.k), db = (uint32_t)(half * p.ug_ld_d * 2);
                mbar_arrive_expect_tx(&R.full[s], 2 * (qb + db));
                bulk_g2s(R.qs(s), p.ug_q + grow * p.k, qb, &R.full[s]);
                bulk_g2s(R.d(s), p.ug_d + grow * p.ug_ld_d, db, &R.full[s]);
                bulk_g2s(R.qs(s) + (size_t)half * p.k, p.ug_q + urow * p.k, qb, &R.full[s]);
                bulk_g2s(R.d(s) + (size_t)half * p.ug_ld_d, p.ug_d + urow * p.ug_ld_d, db,
                         &R.full[s]);
                if (R.raw_rows > 0) jobs(t, 1);
            }
            for (int64_t u = ub0; u < ub1; ++u) {  // phase B: down rows of every expert
                const int r0 = (int)u * kLayerNrb;
                const int nrv = min(kLayerNrb, p.k - r0);
                for (int sg = 0; sg < sg_per_unit; ++sg, ++it) {
                    const int s = it % R.stages;
                    if (it >= R.stages)
                        mbar_wait(&R.empty[s], (it / R.stages - 1) & 1, &g_err_layer);
                    const int ne = min(kCW, n_exp - sg * kCW);
                    const uint32_t qb = (uint32_t)(nrv * p.n_ff), db = (uint32_t)(nrv * p.dn_ld_d * 2);
                    mbar_arrive_expect_tx(&R.full[s], (uint32_t)ne * (qb + db));
                    for (int j = 0; j < ne; ++j) {
                        const int64_t row = (int64_t)expert(sg * kCW + j) * p.dn_stride + r0;
                        bulk_g2s(R.qs(s) + (size_t)j * kLayerNrb * p.n_ff, p.dn_q + row * p.n_ff,
                                 qb, &R.full[s]);
                        bulk_g2s(R.d(s) + (size_t)j * kLayerNrb * p.dn_ld_d,
                                 p.dn_d + row * p.dn_ld_d, db, &R.full[s]);
                    }
                }
            }
            const int first = it > R.stages ? it - R.stages : 0;
            for (int j = first; j < it; ++j)
                mbar_wait(&R.full[j % R.stages], (j / R.stages) & 1, &g_err_layer);
        }
        return;
    }

    // ---------------- consumers, phase A: h = silu(gate . x) * (up . x)
    const XStage xs{reinterpret_cast<int8_t *>(smem + p.plan.off_xq),
                    reinterpret_cast<float *>(smem + p.plan.off_xd)};
    int it = 0, staged_mi = -1, staged_grp = -1;
    XJobs J;
    for (int64_t t = ta0; t < ta1; ++t, ++it) {
        const int s = it % R.stages;
        mbar_wait(&R.full[s], (it / R.stages) & 1, &g_err_layer);
        Q8_TRACE(6);
        const int mi = (int)(t / tpm), ti = (int)(t % tpm);
        const int e = expert(mi);
        const int cnt = tab[p.lay_count + e];
        const int32_t *plist = tab + p.lay_pairs + tab[p.lay_offset + e];
        const int r0 = ti * half;
        const int n_grp = (cnt + xmax - 1) / xmax;
        for (int grp = 0; grp < n_grp; ++grp) {
            const int x0 = grp * xmax;
            const int nx = min(xmax, cnt - x0);
            if (mi != staged_mi || grp != staged_grp) {
                if (staged_mi >= 0) named_bar_sync(kBarConsumers, kCT);
                stage_job_f32(R, J, xs, p.x, p.k, nx,
                              [&](int j) { return plist[x0 + j] / p.n_used; }, &g_err_layer);
                named_bar_sync(kBarConsumers, kCT);
                Q8_TRACE(7);
                staged_mi = mi;
                staged_grp = grp;
            }
            for (int tg = 0; tg < nx; tg += NT) {
                const int n = min(NT, nx - tg);
                with_nt<NT>(n, [&](auto ntc) {
                    constexpr int NTC = decltype(ntc)::value;
                    warp_pairs<NTC>(R.qs(s), R.d(s), p.k, (int)p.ug_ld_d, ga, half, xs, tg, n,
                                    [&](int row, int tt, float gv, float uv) {
                                        if (tt < n) {
                                            const int pr = plist[x0 + tg + tt];
                                            p.h[(int64_t)pr * p.n_ff + r0 + row] =
                                                gv / (1.0f + expf(-gv)) * uv;
                                        }
                                    });
                });
                Q8_TRACE(8);
            }
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&R.empty[s]);
    }

    // ---------------- every CTA's h is written
    named_bar_sync(kBarConsumers, kCT);
    Q8_TRACE(12);
    if (threadIdx.x == 0) grid_barrier(p.bar, gridDim.x, &g_err_layer);
    named_bar_sync(kBarConsumers, kCT);
    Q8_TRACE(11);

    // every pair's h as Q8_0, in grouped (expert, pair) order
    const int P = p.n_tok * p.n_used;
    const int n_valid = tab[p.lay_offset + p.n_mat];
    const XStage hs{reinterpret_cast<int8_t *>(smem + p.off_hq),
                    reinterpret_cast<float *>(smem + p.off_hd)};
    int *inv = reinterpret_cast<int *>(smem + p.off_inv);
    float *ybuf = reinterpret_cast<float *>(smem + p.off_y);
    stage_f32_l2(hs, p.h, p.n_ff, n_valid, [&](int j) { return tab[p.lay_pairs + j]; });
    for (int i = threadIdx.x; i < P; i += kCT) inv[i] = -1;
    named_bar_sync(kBarConsumers, kCT);
    for (int j = threadIdx.x; j < n_valid; j += kCT) inv[tab[p.lay_pairs + j]] = j;
    named_bar_sync(kBarConsumers, kCT);
    Q8_TRACE(7);

    // ---------------- phase B: y = down . hq, out = sum_s p y
    const Geo gb{kLayerNrb * kCW, 1, kLayerNrb};
    for (int64_t u = ub0; u < ub1; ++u) {
        const int r0 = (int)u * kLayerNrb;
        const int nrv = min(kLayerNrb, p.k - r0);
        for (int sg = 0; sg < sg_per_unit; ++sg, ++it) {
            const int s = it % R.stages;
            mbar_wait(&R.full[s], (it / R.stages) & 1, &g_err_layer);
            Q8_TRACE(6);
            const int mi = sg * kCW + warp;
            if (mi < n_exp) {
                const int e = expert(mi);
                const int cnt = tab[p.lay_count + e];
                const int off = tab[p.lay_offset + e];
                // at most 2 activation rows per pass here: 8 rows per warp
                for (int tg = 0; tg < cnt; tg += 2) {
                    const int n = min(2, cnt - tg);
                    with_nt<2>(n, [&](auto ntc) {
                        constexpr int NTC = decltype(ntc)::value;
                        warp_rows<NTC>(R.qs(s), R.d(s), p.n_ff, (int)p.dn_ld_d, gb, hs, off + tg, n,
                                       [&](int row, int tt, float v) {
                                           const int rr = row - warp * kLayerNrb;
                                           if (tt < n && rr < nrv)
                                               ybuf[(off + tg + tt) * kLayerNrb + rr] = v;
                                       });
                    });
                }
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(&R.empty[s]);
            Q8_TRACE(8);
        }
        named_bar_sync(kBarConsumers, kCT);
        for (int i = threadIdx.x; i < p.n_tok * nrv; i += kCT) {
            const int t = i / nrv;
            const int rr = i - t * nrv;
            float acc = 0.0f;
            for (int s2 = 0; s2 < p.n_used; ++s2) {
                const int q = inv[t * p.n_used + s2];
                acc = fmaf(p.route_w[t * p.n_used + s2], q >= 0 ? ybuf[q * kLayerNrb + rr] : 0.0f,
                           acc);
            }
            p.out[(int64_t)t * p.k + r0 + rr] = acc;
        }
        named_bar_sync(kBarConsumers, kCT);
        Q8_TRACE(10);
    }
}

// Whether the fused layer kernel serves this call (the caller checked the
// tensors): routed, at most kLayerMaxPairs pairs, whole-row up/gate tiles.
bool layer_eligible(const q8_tensor *up_gate, const q8_tensor *down, int64_t n_tok,
                    int32_t n_used) {
    const int64_t n_ff = up_gate->rows / 2;
    return n_tok * n_used <= kLayerMaxPairs && up_gate->n_mat <= kCtaGroupMaxMats &&
           up_gate->k <= 4096 && n_ff <= 2048 && n_ff % 16 == 0 && down->k == n_ff;
}

q8_status launch_layer(const q8_tensor *up_gate, const q8_tensor *down, const float *x,
                       int64_t n_tok, const int32_t *ids, const float *route_w, int32_t n_used,
                       float *out, float *h, unsigned *bar, int32_t *err_out, cudaStream_t s) {
    const int64_t P = n_tok * n_used;
    const int64_t n_ff = up_gate->rows / 2;
    LayerParams p{};
    p.ug_q = up_gate->qs;
    p.ug_d = up_gate->d;
    p.ug_ld_d = up_gate->ld_d;
    p.ug_stride = up_gate->mat_stride;
    p.dn_q = down->qs;
    p.dn_d = down->d;
    p.dn_ld_d = down->ld_d;
    p.dn_stride = down->mat_stride;
    p.k = (int)up_gate->k;
    p.n_ff = (int)n_ff;
    p.x = x;
    p.ids = ids;
    p.route_w = route_w;
    p.out = out;
    p.h = h;
    p.bar = bar;
    p.err_out = err_out;
    p.n_tok = (int)n_tok;
    p.n_used = n_used;
    p.n_mat = (int)up_gate->n_mat;
    const GroupLayout L = group_layout(P, up_gate->n_mat);
    p.lay_count = L.count;
    p.lay_offset = L.offset;
    p.lay_list = L.list_small;
    p.lay_big = L.list_big;
    p.lay_pairs = L.pairs;
    // phase-B areas after the grouping tables (all in the plan's table region)
    const int nb_ff = (int)(n_ff / QK);
    int o = (int)L.words * 4;
    o = (o + 15) / 16 * 16;
    const int hq_off = o;
    o += (int)(P * n_ff);
    const int hd_off = o;
    o += (int)(P * nb_ff * 4);
    const int y_off = o;
    o += (int)(P * kLayerNrb * 4);
    const int inv_off = o;
    o += (int)(P * 4);
    const int tab_words = (o + 3) / 4;
    const Geo ga = geo_pair_for_k(p.k);
    int tq = ga.nr * p.k, td = (int)(ga.nr * up_gate->ld_d * 2);
    tq = std::max(tq, kLayerNrb * kCW * p.n_ff);
    td = std::max(td, (int)(kLayerNrb * kCW * down->ld_d * 2));
    if (!make_plan_ctas(tq, td, p.k, (int)std::min<int64_t>(n_tok, kMaxXRows), kLayerNT, 1,
                        &p.plan, tab_words, aligned16(x)) ||
        p.plan.stages < 2)
        Q8_FAIL(Q8_E_UNSUPPORTED, "moe layer: does not fit the shared-memory plan");
    p.off_hq = p.plan.off_tab + hq_off;
    p.off_hd = p.plan.off_tab + hd_off;
    p.off_y = p.plan.off_tab + y_off;
    p.off_inv = p.plan.off_tab + inv_off;

    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64)
        Q8_FAIL(Q8_E_CUDA, "moe layer: no current device");
    auto kern = moe_layer_kernel<kLayerNT>;
    if (!smem_opted_in((const void *)kern, dev)) {
        cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             kSmemLimit);
        if (e != cudaSuccess)
            Q8_FAIL(Q8_E_CUDA, "moe layer: shared-memory attribute: %s", cudaGetErrorString(e));
        set_smem_opted_in((const void *)kern, dev);
    }
    cudaLaunchConfig_t cfg{};
    cfg.gridDim = dim3((unsigned)num_sms());
    cfg.blockDim = dim3(kThreadsStream);
    cfg.dynamicSmemBytes = (size_t)p.plan.bytes;
    cfg.stream = s;
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeCooperative;
    attr[0].val.cooperative = 1;
    attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[1].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 2;
    cudaError_t e = cudaLaunchKernelEx(&cfg, kern, p);
    if (e != cudaSuccess) Q8_FAIL(Q8_E_CUDA, "moe layer: launch: %s", cudaGetErrorString(e));
    return Q8_OK;
}

}  // namespace q8
