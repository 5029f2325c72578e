// q8_route.cu -- the router: the step before the MoE path, which turns a
// token's activations into the routing ids and routing weights that the
// routed calls take as inputs.  The news.hada.io article on Gemma 4 26B-A4B
// names MoE routing only as a run-time option (its opening section on the
// 2016-Xeon set-up, 「CPUを考慮したMoEルーティング」); the reading here is the
// plain top-k router:
//   logits[t][e] = sum_i w_router[e][i] * x[t][i], every product and sum in
//                  fp64 (fp32 inputs; each product is exact in fp64);
//   ids[t]       = the n_used experts with the largest logits, largest first,
//                  equal logits taken by ascending expert index;
//   route_w[t]   = softmax over the selected logits only (the largest one
//                  subtracted before exp, fp64), stored as fp32.
//
// One thread-block cluster per group of up to kRouteTok tokens: the
// cluster's CTAs split the experts (CTA r takes experts e = r, r + C, ...; a
// warp per expert row, 16-byte loads, fp64 fma per token, a fixed xor tree),
// keep the logits in their own shared memory, and after a cluster barrier
// CTA 0 reads every logit through distributed shared memory; a second cluster
// barrier keeps every CTA's shared memory alive until then.  CTA 0 then
// selects the top n_used per token (one warp per token, repeated warp argmax)
// and forms the weights.  The group's activations are staged once as fp64
// (exact), so the inner loop is one fp64 fma per weight and token plus one
// conversion per weight.  No atomics, no global scratch: the results are
// deterministic.
#include <cooperative_groups.h>

#include <algorithm>
#include <cmath>

#include "q8_internal.h"
#include "q8_ptx.cuh"

namespace cg = cooperative_groups;

namespace q8 {

constexpr int kRouteTok = 4;         // most tokens per cluster
constexpr int kRouteThreads = 512;   // most threads per CTA (16 warps)
constexpr int kRouteCluster = 8;     // CTAs per cluster (portable size)
constexpr int kRouteUnroll = 8;      // router-row loads in flight per lane
constexpr int kSmemLimitRoute = 227 * 1024;

struct RouteParams {
    const float *w;  // [n_exp][n_embd]
    const float *x;  // [n_tok][n_embd]
    int n_tok, n_embd, n_exp, n_used;
    int tpc;         // tokens per cluster (1..kRouteTok; fewer when n_embd is long)
    int32_t *ids;    // [n_tok][n_used]
    float *route_w;  // [n_tok][n_used]
    double *logits;  // [n_tok][n_exp] or nullptr
    int off_lg;      // shared-memory offset (bytes) of the logits
};

// Larger logit first; equal logits by the lower expert index (a total order
// on (value, index); NaN logits count as -infinity, so the order stays total).
__device__ __forceinline__ bool route_before(double a, int ia, double b, int ib) {
    return a > b || (a == b && ia < ib);
}

__global__ void __launch_bounds__(kRouteThreads, 1) route_kernel(const __grid_constant__ RouteParams p) {
    extern __shared__ __align__(16) unsigned char smem[];
    cg::cluster_group cluster = cg::this_cluster();
    const int rank = (int)cluster.block_rank();
    const int C = (int)cluster.num_blocks();
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int t0 = (int)(blockIdx.x / C) * p.tpc;
    const int nt = min(p.tpc, p.n_tok - t0);
    // x of token t as fp64 pairs: element 4c, 4c+1 at xa[t * n4 + c], 4c+2,
    // 4c+3 at xb[t * n4 + c] (lane-consecutive 16-byte loads, no bank conflicts)
    const int n4 = p.n_embd / 4;
    double2 *xa = reinterpret_cast<double2 *>(smem);
    double2 *xb = xa + (size_t)p.tpc * n4;
    double *lg = reinterpret_cast<double *>(smem + p.off_lg);  // [tpc][n_exp], own experts only
    const int n_warps = (int)(blockDim.x >> 5);
    Q8_TRACE(0);
    griddep_wait();  // x may come from the preceding kernel
    griddep_launch_dependents();
    for (int i = threadIdx.x; i < nt * n4; i += blockDim.x) {
        const int t = i / n4, c = i - t * n4;
        const float4 v = reinterpret_cast<const float4 *>(p.x + (int64_t)(t0 + t) * p.n_embd)[c];
        xa[i] = make_double2((double)v.x, (double)v.y);
        xb[i] = make_double2((double)v.z, (double)v.w);
    }
    __syncthreads();
    Q8_TRACE(1);
    // logits of this CTA's experts: warp per expert row
    for (int e = rank + C * warp; e < p.n_exp; e += C * n_warps) {
        const float4 *wr = reinterpret_cast<const float4 *>(p.w + (int64_t)e * p.n_embd);
        double acc[kRouteTok];
#pragma unroll
        for (int t = 0; t < kRouteTok; ++t) acc[t] = 0.0;
        // kRouteUnroll row loads in flight per lane, then their products in
        // order (a fixed order per n_embd: the sums are deterministic)
        for (int c0 = lane; c0 < n4; c0 += 32 * kRouteUnroll) {
            float4 wv[kRouteUnroll];
#pragma unroll
            for (int u = 0; u < kRouteUnroll; ++u)
                wv[u] = c0 + 32 * u < n4 ? __ldg(wr + c0 + 32 * u) : make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
            for (int u = 0; u < kRouteUnroll; ++u) {
                const int c = c0 + 32 * u;
                if (c >= n4) break;
                const double w0 = wv[u].x, w1 = wv[u].y, w2 = wv[u].z, w3 = wv[u].w;
#pragma unroll
                for (int t = 0; t < kRouteTok; ++t) {
                    if (t < nt) {
                        const double2 a = xa[t * n4 + c], b = xb[t * n4 + c];
                        acc[t] = fma(w0, a.x, acc[t]);
                        acc[t] = fma(w1, a.y, acc[t]);
                        acc[t] = fma(w2, b.x, acc[t]);
                        acc[t] = fma(w3, b.y, acc[t]);
                    }
                }
            }
        }
#pragma unroll
        for (int t = 0; t < kRouteTok; ++t) {
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) acc[t] += __shfl_xor_sync(0xffffffffu, acc[t], o);
        }
        if (lane == 0) {
#pragma unroll
            for (int t = 0; t < kRouteTok; ++t)
                if (t < nt) lg[t * p.n_exp + e] = acc[t];
        }
    }
    Q8_TRACE(2);
    cluster.sync();  // every CTA's logits are written (release / acquire)
    Q8_TRACE(3);
    if (p.logits) {
        for (int i = threadIdx.x; i < nt * p.n_exp; i += blockDim.x) {
            const int t = i / p.n_exp, e = i - t * p.n_exp;
            if (e % C == rank) p.logits[(int64_t)(t0 + t) * p.n_exp + e] = lg[i];
        }
    }
    if (rank == 0) {
        // gather the other CTAs' logits into this CTA's array (each expert's
        // slot is written by exactly one CTA; this CTA's own slots stay)
        for (int i = threadIdx.x; i < nt * p.n_exp; i += blockDim.x) {
            const int e = i % p.n_exp;
            if (e % C != 0) lg[i] = cluster.map_shared_rank(lg, e % C)[i];
        }
        __syncthreads();
    }
    Q8_TRACE(4);
    cluster.sync();  // CTA 0 is done reading the others' shared memory
    Q8_TRACE(5);
    if (rank == 0 && warp < nt) {
        // token t0 + warp: repeated warp argmax over the not-yet-selected
        // experts.  Lane l owns experts l, l + 32, ... (at most 32: n_exp <=
        // 1024) and keeps its best unselected one in registers; each round
        // the warp's best is the next selection, and only its owner lane
        // looks at its candidates again.
        const int t = warp;
        auto logit = [&](int e) -> double {  // NaN ranks as -infinity
            const double v = lg[t * p.n_exp + e];
            return v != v ? -INFINITY : v;
        };
        uint32_t taken = 0;  // bit c: expert lane + 32 c is selected
        double lv = -INFINITY;
        int li = p.n_exp;  // this lane's best unselected expert (n_exp: none)
        auto rescan = [&]() {
            lv = -INFINITY;
            li = p.n_exp;
            for (int e = lane, c = 0; e < p.n_exp; e += 32, ++c) {
                if ((taken >> c) & 1u) continue;
                const double v = logit(e);
                if (li == p.n_exp || route_before(v, e, lv, li)) {
                    lv = v;
                    li = e;
                }
            }
        };
        rescan();
        double first = 0.0, mine = -INFINITY;  // lane k keeps the k-th selected logit
        for (int k = 0; k < p.n_used; ++k) {
            double bv = lv;
            int bi = li;
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) {
                const double ov = __shfl_xor_sync(0xffffffffu, bv, o);
                const int oi = __shfl_xor_sync(0xffffffffu, bi, o);
                if (oi < p.n_exp && (bi == p.n_exp || route_before(ov, oi, bv, bi))) {
                    bv = ov;
                    bi = oi;
                }
            }
            // n_used <= n_exp: some expert is always left, so bi < n_exp, and
            // every lane holds the same (bv, bi)
            if (lane == 0) p.ids[(int64_t)(t0 + t) * p.n_used + k] = bi;
            if (k == 0) first = bv;
            if (lane == k) mine = bv;
            if ((bi & 31) == lane) {
                taken |= 1u << (bi >> 5);
                rescan();
            }
            __syncwarp();
        }
        Q8_TRACE(6);
        // softmax over the selected logits (largest first), fp64
        const double ex = lane < p.n_used ? exp(mine - first) : 0.0;
        double sum = ex;
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
        if (lane < p.n_used) p.route_w[(int64_t)(t0 + t) * p.n_used + lane] = (float)(ex / sum);
        Q8_TRACE(7);
    }
}

}  // namespace q8

using namespace q8;

extern "C" q8_status q8_route(const float *w_router, const float *x, int64_t n_tok,
                              int64_t n_embd, int64_t n_exp, int32_t n_used, int32_t *ids,
                              float *route_w, double *logits, void *stream) {
    const char *fn = "q8_route";
    Q8_REQUIRE(w_router && x && ids && route_w, Q8_E_NULL, "%s: NULL pointer", fn);
    Q8_REQUIRE(n_tok >= 1 && n_tok <= (1LL << 24), Q8_E_SHAPE, "%s: n_tok=%lld", fn,
               (long long)n_tok);
    Q8_REQUIRE(n_embd >= 4 && n_embd % 4 == 0 && n_embd <= Q8_MAX_K, Q8_E_SHAPE,
               "%s: n_embd=%lld must be a multiple of 4 in [4, %d]", fn, (long long)n_embd,
               Q8_MAX_K);
    Q8_REQUIRE(n_exp >= 1 && n_exp <= Q8_ROUTE_MAX_EXP, Q8_E_SHAPE, "%s: n_exp=%lld (1..%d)", fn,
               (long long)n_exp, Q8_ROUTE_MAX_EXP);
    Q8_REQUIRE(n_used >= 1 && n_used <= Q8_MAX_USED && n_used <= n_exp, Q8_E_SHAPE,
               "%s: n_used=%d (1..min(n_exp, %d))", fn, n_used, Q8_MAX_USED);
    Q8_REQUIRE(aligned16(w_router) && aligned16(x), Q8_E_ALIGN,
               "%s: w_router and x must be 16-byte aligned", fn);
    Q8_REQUIRE(((uintptr_t)ids & 3u) == 0 && ((uintptr_t)route_w & 3u) == 0 &&
                   ((uintptr_t)logits & 7u) == 0,
               Q8_E_ALIGN, "%s: ids/route_w/logits misaligned", fn);
    RouteParams p{};
    p.w = w_router;
    p.x = x;
    p.n_tok = (int)n_tok;
    p.n_embd = (int)n_embd;
    p.n_exp = (int)n_exp;
    p.n_used = n_used;
    p.ids = ids;
    p.route_w = route_w;
    p.logits = logits;
    const int C = kRouteCluster;
    // tokens per cluster: as many as fit (up to kRouteTok), the fp64 rows of
    // x and the logits of each
    const int per_tok = (int)n_embd * 8 + (int)n_exp * 8 + 32;
    p.tpc = std::min<int>(kRouteTok, kSmemLimitRoute / per_tok);
    Q8_REQUIRE(p.tpc >= 1, Q8_E_UNSUPPORTED, "%s: shared-memory plan too large", fn);
    const int x_bytes = p.tpc * (int)n_embd * 8;  // two double2 arrays (xa, xb)
    p.off_lg = (x_bytes + 15) / 16 * 16;
    const int lg_bytes = p.tpc * (int)n_exp * 8;
    const int smem = p.off_lg + lg_bytes;
    Q8_REQUIRE(smem <= kSmemLimitRoute, Q8_E_UNSUPPORTED, "%s: shared-memory plan too large", fn);
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64)
        Q8_FAIL(Q8_E_CUDA, "%s: no current device", fn);
    if (!smem_opted_in((const void *)route_kernel, dev)) {
        cudaError_t e = cudaFuncSetAttribute(route_kernel,
                                             cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             kSmemLimitRoute);
        if (e != cudaSuccess)
            Q8_FAIL(Q8_E_CUDA, "%s: shared-memory attribute: %s", fn, cudaGetErrorString(e));
        set_smem_opted_in((const void *)route_kernel, dev);
    }
    const int groups = (int)((n_tok + p.tpc - 1) / p.tpc);
    // a few clusters (decode): 16 warps per CTA, one router row each at 128
    // experts; many: 8 warps, so that two CTAs share an SM
    const int threads = (int64_t)groups * C * 2 <= num_sms() ? kRouteThreads : kRouteThreads / 2;
    cudaLaunchConfig_t cfg{};
    cfg.gridDim = dim3((unsigned)(groups * C));
    cfg.blockDim = dim3((unsigned)threads);
    cfg.dynamicSmemBytes = (size_t)smem;
    cfg.stream = (cudaStream_t)stream;
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = C;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[1].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 2;
    cudaError_t e = cudaLaunchKernelEx(&cfg, route_kernel, p);
    if (e != cudaSuccess) Q8_FAIL(Q8_E_CUDA, "%s: launch: %s", fn, cudaGetErrorString(e));
    return Q8_OK;
}
