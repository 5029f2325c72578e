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
// The raw x slot and the phase-B areas share one region: x is staged before
// phase B starts.
//  phase A  tiles of 8 gate rows + the 8 matching up rows of one routed
//           expert (k <= 4096: whole rows per warp); x rows are copied by the
//           producer and quantized in shared memory; h goes to global memory.
//  barrier  all CTAs' h is written (bounded wait).
//  phase B  units of nrb (8) down rows; a stage holds those rows of up to 8
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

q8_status clear_wait_errors_layer() {
    const int zero = 0;
    cudaError_t e = cudaMemcpyToSymbol(g_err_layer, &zero, sizeof(int));
    return e == cudaSuccess ? Q8_OK : Q8_E_CUDA;
}

constexpr int kLayerNT = 4;   // activation rows per pass (template bound), several tokens
// The h bulk copy's mbarrier: after the ring's barriers in the plan's first
// 256 bytes (full and empty of kMaxStages stages, then the raw slot's two).
constexpr int kLayerHBar = 2 * kMaxStages * 8 + 16;
static_assert(kLayerHBar + 8 <= 256, "barrier area");
// fp32 h of all pairs is copied back in bulk when it takes at most this much
// shared memory (the copy shares the phase-B region with the other areas)
constexpr int kLayerHBulkBytes = 24 * 1024;

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
    unsigned *bar;  // grid barrier: 64-bit arrival counter (8-byte aligned)
    int32_t *err_out;
    int n_tok, n_used, n_mat;
    int64_t lay_count, lay_offset, lay_list, lay_big, lay_pairs;
    int off_hq, off_hd, off_y, off_inv;  // phase-B areas
    int off_hf;                          // fp32 h of all pairs, copied in bulk (-1: none)
    int off_rw;                          // the routing weights [P], staged at the start
    int nrb;                             // down rows per unit
    Plan plan;
};

__device__ __forceinline__ unsigned long long ld_acquire_u64(const unsigned long long *p) {
    unsigned long long v;
    asm volatile("ld.acquire.gpu.global.u64 %0, [%1];" : "=l"(v) : "l"(p) : "memory");
    return v;
}

// Barrier of all n CTAs of a co-resident grid, entered by one thread per CTA
// after its CTA's global writes (ordered by a CTA barrier before the call).
// bar: a 64-bit arrival counter (8-byte aligned) that only grows: every
// launch of n CTAs adds n, so between launches it is a multiple of n (zero
// before the first use).  A CTA adds one (release) and waits (acquire) until
// the counter reaches the next multiple of n above its own arrival: one
// atomic per CTA and no reset, so the last arrival releases the others with
// its own atomic.  The add is acquire-release at GPU scope and the polls are
// acquire loads: the adds form one release sequence, so a CTA that reads the
// final count has seen every CTA's writes before its arrival (the CTA
// barrier before the call makes them the arriving thread's), with no
// separate fences.
// Bounded: after limit_ns the wait records Q8_WAIT_TIMEOUT and returns
// false (the counter is then left off its multiple: q8_check reports it).
__device__ __forceinline__ unsigned long long atom_add_acq_rel_u64(unsigned long long *p,
                                                                   unsigned long long v) {
    unsigned long long old;
    asm volatile("atom.acq_rel.gpu.global.add.u64 %0, [%1], %2;" : "=l"(old) : "l"(p), "l"(v)
                 : "memory");
    return old;
}

__device__ __forceinline__ bool grid_barrier(unsigned *bar, unsigned n, int *err,
                                             uint64_t limit_ns = kWaitLimitNs) {
    unsigned long long *cnt = reinterpret_cast<unsigned long long *>(bar);
    const unsigned long long old = atom_add_acq_rel_u64(cnt, 1ull);
    const unsigned long long target = (old / n + 1) * n;
    if (old + 1 == target) return true;
    const uint64_t t0 = globaltimer_ns();
    while (ld_acquire_u64(cnt) < target) {
        if (globaltimer_ns() - t0 > limit_ns) {
            atomicOr(err, Q8_WAIT_TIMEOUT);
            return false;
        }
        __nanosleep(32);
    }
    return true;
}

// Make this thread's global writes visible to later bulk (async-proxy) reads
// of the same memory, and order its later bulk reads after what it observed.
__device__ __forceinline__ void fence_proxy_async_global() {
    asm volatile("fence.proxy.async.global;" ::: "memory");
}

// Quantize fp32 rows written in this launch by other CTAs (so loaded at L2,
// not through L1): n rows of k floats, row j at src + arow(j) * k, into the
// stage, one thread per 32-block.
template <class RowFn>
__device__ __forceinline__ void stage_f32_l2(const XStage &xs, const float *src, int k, int n,
                                             RowFn arow, int tid, int nthr) {
    const int nb = k / QK;
    for (int blk = tid; blk < n * nb; blk += nthr) {
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

// Phase A at one decode token, with x staged once for all experts: a consumer
// group's up/gate tiles in one tight loop, the lane's activation blocks held
// in registers for the whole phase.  The arithmetic and its order are those
// of warp_pairs (dot_rows over gate row row0 + i and up row half + row0 + i,
// then the reduce-scatter tree), so h has the same bits; the per-tile
// dispatch of the generic path is gone.
template <int RPW, int ITERS, int G>
__device__ __forceinline__ void layer_pairs_run(const Ring &R, const XStage &xs,
                                                const LayerParams &p, const int32_t *tab,
                                                int tpm, int half, int ta0, int ta1,
                                                int grp, int w8) {
    const int lane = threadIdx.x & 31;
    const int k = p.k, nb = k / QK, ld_d = (int)p.ug_ld_d;
    const int h0 = ((lane >> 2) & 1) * 16, h1 = 16 - h0;
    constexpr int H = RPW / 2;
    const int row0 = w8 * H;
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
    const int up_idx = idx + H;
    const int up_lane = reduce_scatter_lane<VP>(up_idx < VP ? up_idx : 0);
    const bool writer = (lane & (32 / VP - 1)) == 0 && idx < H;
    for (int t = ta0 + grp; t < ta1; t += G) {
        const int it = t - ta0;
        const int s = it % R.stages;
        mbar_wait(&R.full[s], (it / R.stages) & 1, &g_err_layer);
        Q8_TRACE(6);
        const int mi = (int)(t / tpm), ti = (int)(t % tpm);
        const int e = tab[p.lay_list + mi];
        const int pr = tab[p.lay_pairs + tab[p.lay_offset + e]];  // one pair per expert
        const int r0 = ti * half;
        const int8_t *sq = R.qs(s);
        const uint16_t *sd = R.d(s);
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
                    const int srow = r < H ? row0 + r : half + row0 + (r - H);
                    const int8_t *wp = sq + (size_t)srow * k + kb * QK;
                    w0[r] = *reinterpret_cast<const uint4 *>(wp + h0);
                    w1[r] = *reinterpret_cast<const uint4 *>(wp + h1);
                    dw[r] = scale_value(sd[(size_t)srow * ld_d + kb]);
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
        const float u = __shfl_sync(0xffffffffu, v, up_lane);
        __syncwarp();
        if (lane == 0) mbar_arrive(&R.empty[s]);
        Q8_TRACE(8);
        if (writer) p.h[(int64_t)pr * p.n_ff + r0 + row0 + idx] = v / (1.0f + expf(-v)) * u;
    }
}

// G consumer groups of kCW warps share one ring: group g takes every G-th
// tile of phase A and every G-th unit of phase B (G = 2 doubles the warps
// that hide each other's latency, at one CTA per SM).  G > 1 needs the
// one-token variant (x staged once, shared by the groups).
template <int NT, int G>
__global__ void __launch_bounds__((G * kCW + 1) * 32, 1)
    moe_layer_kernel(const __grid_constant__ LayerParams p) {
    static_assert(G == 1 || NT == 1, "several consumer groups need the one-token variant");
    constexpr int kProd = G * kCW;  // the producer warp
    constexpr int kAll = G * kCT;   // consumer threads
    extern __shared__ __align__(128) unsigned char smem[];
    Q8_TRACE(0);
    const Ring R = ring_init(smem, p.plan);
    // the bulk copy of h after the grid barrier completes on its own mbarrier
    uint64_t *hbar = reinterpret_cast<uint64_t *>(smem + kLayerHBar);
    if (threadIdx.x == 0) {
        mbar_init(hbar, 1);
        fence_barrier_init();
    }
    Q8_TRACE(1);
    griddep_wait();  // x, ids and route_w may come from the preceding kernel
    griddep_launch_dependents();
    Q8_TRACE(2);
    // One token (the NT == 1 variant): every routed expert reads the same x
    // row, so the producer fetches it before the grouping and it is staged
    // once for the whole of phase A.
    const bool x_once = NT == 1 && R.raw_rows > 0;
    if (x_once && threadIdx.x == kProd * 32) {
        mbar_arrive_expect_tx(R.xfull, (uint32_t)p.k * 4);
        bulk_g2s_keep(R.raw, p.x, (uint32_t)p.k * 4, R.xfull);
    }
    // the routing weights are read only by the combine at the very end: their
    // copy starts now, asynchronously (the grouping's read of the ids does not
    // wait behind it), and the issuing threads wait for it before the grid
    // barrier
    float *s_rw = reinterpret_cast<float *>(smem + p.off_rw);
    for (int i = threadIdx.x; i < p.n_tok * p.n_used; i += blockDim.x) cp_async4(s_rw + i, p.route_w + i);
    cp_async_commit();
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
    Q8_TRACE(25);
    const int n_exp = tab[WS_N_SMALL];
    const Geo ga = geo_pair_for_k(p.k);
    const int half = ga.nr / 2;
    const int tpm = p.n_ff / half;
    const int nrb = p.nrb;
    const int units = (p.k + nrb - 1) / nrb;
    const int sg_per_unit = (n_exp + kCW - 1) / kCW;
    const int xmax = p.plan.xmax;
    // this CTA's tiles and units (32-bit: at most 32 experts of 2048 / 8 tiles)
    const int n_tiles_a = n_exp * tpm;
    const int ta0 = (int)((unsigned)n_tiles_a * blockIdx.x / gridDim.x);
    const int ta1 = (int)((unsigned)n_tiles_a * (blockIdx.x + 1) / gridDim.x);
    const int ub0 = (int)((unsigned)units * blockIdx.x / gridDim.x);
    const int ub1 = (int)((unsigned)units * (blockIdx.x + 1) / gridDim.x);
    auto expert = [&](int i) { return tab[p.lay_list + i]; };

    if (warp == kProd) {  // ---------------- producer
        Q8_TRACE(24);
        if (lane == 0) {
            int it = 0;
            XJobs J;
            auto jobs = [&](int t, int when) {
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
            for (int t = ta0; t < ta1; ++t, ++it) {  // phase A: gate/up tiles
                const int s = it % R.stages;
                if (R.raw_rows > 0 && !x_once) jobs(t, 0);
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
                if (R.raw_rows > 0 && !x_once) jobs(t, 1);
            }
            for (int u = ub0; u < ub1; ++u) {  // phase B: down rows of every expert
                const int r0 = (int)u * nrb;
                const int nrv = min(nrb, p.k - r0);
                for (int sg = 0; sg < sg_per_unit; ++sg, ++it) {
                    const int s = it % R.stages;
                    if (it >= R.stages)
                        mbar_wait(&R.empty[s], (it / R.stages - 1) & 1, &g_err_layer);
                    const int ne = min(kCW, n_exp - sg * kCW);
                    const uint32_t qb = (uint32_t)(nrv * p.n_ff), db = (uint32_t)(nrv * p.dn_ld_d * 2);
                    mbar_arrive_expect_tx(&R.full[s], (uint32_t)ne * (qb + db));
                    for (int j = 0; j < ne; ++j) {
                        const int64_t row = (int64_t)expert(sg * kCW + j) * p.dn_stride + r0;
                        bulk_g2s(R.qs(s) + (size_t)j * nrb * p.n_ff, p.dn_q + row * p.n_ff,
                                 qb, &R.full[s]);
                        bulk_g2s(R.d(s) + (size_t)j * nrb * p.dn_ld_d,
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

    // ---------------- consumers
    const int grp = warp / kCW;  // consumer group
    const int w8 = warp % kCW;   // warp within the group
    const int bar_grp = kBarConsumers + grp;
    const int bar_all = kBarConsumers + G;
    auto sync_grp = [&]() { named_bar_sync(bar_grp, kCT); };
    auto sync_all = [&]() { named_bar_sync(G == 1 ? kBarConsumers : bar_all, kAll); };

    // phase A: h = silu(gate . x) * (up . x)
    const XStage xs{reinterpret_cast<int8_t *>(smem + p.plan.off_xq),
                    reinterpret_cast<float *>(smem + p.plan.off_xd)};
    int staged_mi = -1, staged_grp = -1;
    XJobs J;
    if (x_once) {
        mbar_wait(R.xfull, 0, &g_err_layer);
        stage_f32_smem_tpb<2>(xs, R.raw, p.k, 1, [](int j) { return j; }, threadIdx.x, kAll);
        sync_all();
        Q8_TRACE(7);
    }
    bool phase_a_done = false;
    if constexpr (NT == 1) {
        if (x_once) {
            // one decode token: every expert has one pair and reads the one
            // staged x row
            const int iters = (p.k / QK + 31) / 32;
            if (ga.rpw == 2 && iters == 1)
                layer_pairs_run<2, 1, G>(R, xs, p, tab, tpm, half, ta0, ta1, grp, w8);
            else if (ga.rpw == 2 && iters == 2)
                layer_pairs_run<2, 2, G>(R, xs, p, tab, tpm, half, ta0, ta1, grp, w8);
            else if (ga.rpw == 2 && iters == 3)
                layer_pairs_run<2, 3, G>(R, xs, p, tab, tpm, half, ta0, ta1, grp, w8);
            else if (ga.rpw == 2)
                layer_pairs_run<2, 4, G>(R, xs, p, tab, tpm, half, ta0, ta1, grp, w8);
            else
                layer_pairs_run<4, 1, G>(R, xs, p, tab, tpm, half, ta0, ta1, grp, w8);
            phase_a_done = true;
        }
    }
    for (int t = ta0 + grp; t < ta1 && !phase_a_done; t += G) {
        const int it = t - ta0;
        const int s = it % R.stages;
        mbar_wait(&R.full[s], (it / R.stages) & 1, &g_err_layer);
        Q8_TRACE(6);
        const int mi = (int)(t / tpm), ti = (int)(t % tpm);
        const int e = expert(mi);
        const int cnt = tab[p.lay_count + e];
        const int32_t *plist = tab + p.lay_pairs + tab[p.lay_offset + e];
        const int r0 = ti * half;
        const int n_grp = (cnt + xmax - 1) / xmax;
        for (int xg = 0; xg < n_grp; ++xg) {
            const int x0 = xg * xmax;
            const int nx = min(xmax, cnt - x0);
            if (!x_once && (mi != staged_mi || xg != staged_grp)) {
                // (G == 1 here)
                if (staged_mi >= 0) sync_grp();
                stage_job_f32(R, J, xs, p.x, p.k, nx,
                              [&](int j) { return plist[x0 + j] / p.n_used; }, &g_err_layer);
                sync_grp();
                Q8_TRACE(7);
                staged_mi = mi;
                staged_grp = xg;
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
                                    },
                                    w8);
                });
                Q8_TRACE(8);
            }
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&R.empty[s]);
    }

    // ---------------- every CTA's h is written
    const int P = p.n_tok * p.n_used;
    cp_async_wait<0>();  // this thread's part of the routing weights has landed
    if (p.off_hf >= 0) fence_proxy_async_global();  // h is read back by a bulk copy
    sync_all();
    Q8_TRACE(12);
    if (threadIdx.x == 0) {
        grid_barrier(p.bar, gridDim.x, &g_err_layer);
        if (p.off_hf >= 0) {
            // all pairs' h [P][n_ff] in one bulk copy (16-byte aligned, a
            // multiple of 16 bytes): one request stream instead of a load per
            // thread, each waiting behind the weight stream
            fence_proxy_async_global();
            const uint32_t bytes = (uint32_t)P * (uint32_t)p.n_ff * 4u;
            mbar_arrive_expect_tx(hbar, bytes);
            bulk_g2s_keep(smem + p.off_hf, p.h, bytes, hbar);
        }
    }
    sync_all();
    Q8_TRACE(11);

    // every pair's h as Q8_0, in grouped (expert, pair) order
    const int n_valid = tab[p.lay_offset + p.n_mat];
    const XStage hs{reinterpret_cast<int8_t *>(smem + p.off_hq),
                    reinterpret_cast<float *>(smem + p.off_hd)};
    int *inv = reinterpret_cast<int *>(smem + p.off_inv);
    float *ybuf = reinterpret_cast<float *>(smem + p.off_y) + (size_t)grp * P * nrb;
    if (p.off_hf >= 0) {
        mbar_wait(hbar, 0, &g_err_layer);
        Q8_TRACE(14);
        stage_f32_smem_tpb<2>(hs, reinterpret_cast<const float *>(smem + p.off_hf), p.n_ff,
                              n_valid, [&](int j) { return tab[p.lay_pairs + j]; }, threadIdx.x,
                              kAll);
        Q8_TRACE(16);
    } else {
        stage_f32_l2(hs, p.h, p.n_ff, n_valid, [&](int j) { return tab[p.lay_pairs + j]; },
                     threadIdx.x, kAll);
    }
    // inv[pair] = its position in the grouped order (-1: an invalid pair);
    // at most kLayerMaxPairs pairs, so one pass of a short scan
    for (int i = threadIdx.x; i < P; i += kAll) {
        int q = -1;
        for (int j = 0; j < n_valid; ++j)
            if (tab[p.lay_pairs + j] == i) q = j;
        inv[i] = q;
    }
    sync_all();
    Q8_TRACE(7);

    // ---------------- phase B: y = down . hq, out = sum_s p y
    const Geo gb{nrb * kCW, 1, nrb};
    const int itb = ta1 - ta0;  // ring position of the first phase-B stage
    const int gtid = threadIdx.x - grp * kCT;
    for (int u = ub0 + grp; u < ub1; u += G) {
        const int r0 = (int)u * nrb;
        const int nrv = min(nrb, p.k - r0);
        for (int sg = 0; sg < sg_per_unit; ++sg) {
            const int it = itb + (u - ub0) * sg_per_unit + sg;
            const int s = it % R.stages;
            mbar_wait(&R.full[s], (it / R.stages) & 1, &g_err_layer);
            Q8_TRACE(6);
            const int mi = sg * kCW + w8;
            if (mi < n_exp) {
                const int e = expert(mi);
                const int cnt = tab[p.lay_count + e];
                const int off = tab[p.lay_offset + e];
                // at most 2 activation rows per pass here (up to 8 rows per
                // warp); one at one token (an expert then has one pair)
                constexpr int NB = NT == 1 ? 1 : 2;
                for (int tg = 0; tg < cnt; tg += NB) {
                    const int n = min(NB, cnt - tg);
                    with_nt<NB>(n, [&](auto ntc) {
                        constexpr int NTC = decltype(ntc)::value;
                        auto emit = [&](int row, int tt, float v) {
                            const int rr = row - w8 * nrb;
                            if (tt < n && rr < nrv) ybuf[(off + tg + tt) * nrb + rr] = v;
                        };
                        if (nrb == 8)
                            warp_rows<NTC, 8>(R.qs(s), R.d(s), p.n_ff, (int)p.dn_ld_d, gb, hs,
                                              off + tg, n, emit, w8);
                        else
                            warp_rows<NTC, 4>(R.qs(s), R.d(s), p.n_ff, (int)p.dn_ld_d, gb, hs,
                                              off + tg, n, emit, w8);
                    });
                }
            }
            Q8_TRACE(13);
            __syncwarp();
            if (lane == 0) mbar_arrive(&R.empty[s]);
            Q8_TRACE(8);
        }
        sync_grp();
        Q8_TRACE(15);
        for (int i = gtid; i < p.n_tok * nrv; i += kCT) {
            const int t = i / nrv;
            const int rr = i - t * nrv;
            float acc = 0.0f;
#pragma unroll 8
            for (int s2 = 0; s2 < p.n_used; ++s2) {
                const int q = inv[t * p.n_used + s2];
                acc = fmaf(s_rw[t * p.n_used + s2], q >= 0 ? ybuf[q * nrb + rr] : 0.0f, acc);
            }
            p.out[(int64_t)t * p.k + r0 + rr] = acc;
        }
        sync_grp();
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

// Shared-memory plan of the layer kernel: barriers, the ring (stages sized
// for the larger of a gate/up tile and a phase-B stage), the x stage, the
// grouping tables, then one region that holds the raw x slot during phase A
// and the phase-B areas (all pairs' hq and scales, y, the pair inverse)
// afterwards.
static bool layer_plan(LayerParams &p, int64_t P, int n_ff, int tq, int td, int xrows, int ctas,
                       int nrb, bool raw, int group_words, int groups) {
    const int budget = smem_budget(ctas);
    const int nb_ff = n_ff / QK;
    const int xmax = xrows;
    const int x_bytes = xmax * p.k + ((xmax * (p.k / QK) * 4 + 15) / 16) * 16;
    const int tab_bytes = ((group_words * 4 + 15) / 16) * 16;
    const int rw_bytes = (int)((P * 4 + 15) / 16 * 16);
    const int raw_rows = raw ? std::min(xmax, kRawSlotBytes / (4 * p.k)) : 0;
    const int raw_bytes = raw_rows * 4 * p.k;
    int o = 0;
    const int hq = o;
    o += (int)(P * n_ff);
    o = (o + 15) / 16 * 16;
    const int hd = o;
    o += (int)(P * nb_ff * 4);
    const int y = o;
    o += (int)(P * nrb * 4) * groups;  // one y buffer per consumer group
    const int inv = o;
    o += (int)(P * 4);
    int hf = -1;
    if (P * n_ff * 4 <= kLayerHBulkBytes) {
        o = (o + 15) / 16 * 16;
        hf = o;
        o += (int)(P * n_ff * 4);
    }
    const int union_bytes = (std::max(o, raw_bytes) + 127) / 128 * 128;
    const int stage_qs = round128(tq);
    const int stage_bytes = stage_qs + round128(td);
    const int fixed = 256 + x_bytes + tab_bytes + rw_bytes + union_bytes;
    int stages = (budget - fixed) / stage_bytes;
    if (stages > kMaxStages) stages = kMaxStages;
    if (stages < 2) return false;
    Plan &pl = p.plan;
    pl = Plan{};
    pl.stages = stages;
    pl.stage_qs = stage_qs;
    pl.stage_bytes = stage_bytes;
    pl.xmax = xmax;
    pl.max_nb = p.k / QK;
    pl.off_full = 0;
    pl.off_empty = kMaxStages * 8;
    pl.off_xfull = 2 * kMaxStages * 8;
    pl.off_xempty = pl.off_xfull + 8;
    pl.off_ring = 256;
    pl.off_xq = pl.off_ring + stages * stage_bytes;
    pl.off_xd = pl.off_xq + xmax * p.k;
    pl.off_part = pl.off_xd + ((xmax * (p.k / QK) * 4 + 15) / 16) * 16;  // unused
    pl.off_tab = pl.off_part;
    pl.tab_words = group_words;
    p.off_rw = pl.off_tab + tab_bytes;
    const int off_union = p.off_rw + rw_bytes;
    pl.raw_rows = raw_rows;
    pl.off_raw = off_union;
    pl.bytes = off_union + union_bytes;
    pl.ctas = ctas;
    p.off_hq = off_union + hq;
    p.off_hd = off_union + hd;
    p.off_y = off_union + y;
    p.off_inv = off_union + inv;
    p.off_hf = hf >= 0 ? off_union + hf : -1;
    p.nrb = nrb;
    return pl.bytes <= budget;
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
    const Geo ga = geo_pair_for_k(p.k);
    const int tq = std::max<int>(ga.nr * p.k, 8 * kCW * p.n_ff);
    const int td = std::max<int>((int)(ga.nr * up_gate->ld_d * 2), (int)(8 * kCW * down->ld_d * 2));
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64)
        Q8_FAIL(Q8_E_CUDA, "moe layer: no current device");
    auto opt_in = [&](void (*kern)(LayerParams)) -> bool {
        if (smem_opted_in((const void *)kern, dev)) return true;
        if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemLimit) !=
            cudaSuccess)
            return false;
        set_smem_opted_in((const void *)kern, dev);
        return true;
    };
    // one CTA per SM with 8-row down units (two CTAs per SM, with half the
    // ring each, measured slower: the ring then holds too little of the
    // stream); one token runs the variant without multi-row passes
    const int xrows = (int)std::min<int64_t>(n_tok, kMaxXRows);
    // one token: two consumer groups (the x row is staged once and shared)
    const int groups = n_tok == 1 && aligned16(x) ? 2 : 1;
    if (!layer_plan(p, P, (int)n_ff, tq, td, xrows, 1, 8, aligned16(x), (int)L.words, groups))
        Q8_FAIL(Q8_E_UNSUPPORTED, "moe layer: does not fit the shared-memory plan");
    void (*kern)(LayerParams) = groups == 2 ? moe_layer_kernel<1, 2> : moe_layer_kernel<kLayerNT, 1>;
    if (!opt_in(kern)) Q8_FAIL(Q8_E_CUDA, "moe layer: shared-memory attribute refused");
    cudaLaunchConfig_t cfg{};
    cfg.gridDim = dim3((unsigned)(num_sms() * p.plan.ctas));
    cfg.blockDim = dim3((unsigned)((groups * kCW + 1) * 32));
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

// Test hook: one bounded wait that cannot succeed.  kind 0: an mbarrier
// phase that nothing completes; kind 1: the grid barrier with one arrival
// short (n = gridDim.x + 1, counter starting at zero).  Both give up after limit_ns, latch
// Q8_WAIT_TIMEOUT in this file's error word and return.
__global__ void wait_probe_kernel(int kind, uint64_t limit_ns, unsigned *bar) {
    __shared__ uint64_t mb;
    if (kind == 0) {
        if (threadIdx.x == 0) {
            mbar_init(&mb, 1);
            fence_barrier_init();
        }
        __syncthreads();
        if (threadIdx.x == 0) mbar_wait_for(&mb, 0, &g_err_layer, limit_ns);
    } else {
        __syncthreads();
        if (threadIdx.x == 0) grid_barrier(bar, gridDim.x + 1, &g_err_layer, limit_ns);
    }
}

}  // namespace q8

using namespace q8;

extern "C" q8_status q8_debug_wait_timeout(int32_t kind, int64_t limit_ns, unsigned *bar,
                                           void *stream) {
    Q8_REQUIRE(kind == 0 || kind == 1, Q8_E_SHAPE, "q8_debug_wait_timeout: kind %d", kind);
    Q8_REQUIRE(limit_ns >= 1000 && limit_ns <= 10000000000LL, Q8_E_SHAPE,
               "q8_debug_wait_timeout: limit_ns=%lld outside [1e3, 1e10]", (long long)limit_ns);
    Q8_REQUIRE(kind == 0 || bar != nullptr, Q8_E_NULL, "q8_debug_wait_timeout: bar is NULL");
    Q8_REQUIRE(((uintptr_t)bar & 7u) == 0, Q8_E_ALIGN,
               "q8_debug_wait_timeout: bar must be 8-byte aligned");
    wait_probe_kernel<<<kind == 0 ? 1 : 2, 32, 0, (cudaStream_t)stream>>>(
        kind, (uint64_t)limit_ns, bar);
    return launch_status("wait_probe_kernel");
}
