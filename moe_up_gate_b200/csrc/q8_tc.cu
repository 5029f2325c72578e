// q8_tc.cu -- the int8 tensor-core (tcgen05) path of the routed matmuls, for
// experts that receive at least kTcMinPairs routed rows: the fused MoE
// up/gate + SwiGLU and the mul_mat_id down projection.  With that many
// activation rows per expert the step is a real (small) dense contraction,
// so it goes to the tensor cores; below that the dp4a streaming kernels serve.
//
// One CTA computes one 128-row weight tile of one expert (up/gate: 64 gate
// rows and the 64 matching up rows) for up to 32 of the expert's routed rows
// at a time:
//  * warp 0 (one lane) streams the tile in 128-byte K chunks (4 Q8_0 blocks)
//    with 2-D tensor (TMA) loads into a ring of 128-byte-swizzled stages;
//  * the activation rows are staged once, as Q8_0, in the canonical no-swizzle
//    K-major layout (8-row x 16-byte core matrices), padded with zero rows to
//    a multiple of 16;
//  * warp 1 (one lane) issues one tcgen05.mma.kind::i8 per Q8_0 block
//    (M=128, N=16..32, K=32): every block's exact int32 dot products land in
//    a tensor-memory slot of their own, because each block has its own pair
//    of scales and the int32 sum cannot run across blocks;
//  * warps 2-9 read each slot back (thread = weight row, 16 activation rows
//    per warp), scale by d_w * d_x in fp32 and accumulate, in block order.
// Every wait is bounded (q8_ptx.cuh); tensor memory is freed before exit.
#include <cuda.h>
#include <cudaTypedefs.h>

#include <algorithm>
#include <mutex>

#include "q8_internal.h"
#include "q8_stream.cuh"
#include "q8_tc.cuh"

namespace q8 {

constexpr int kTcN = 32;            // activation rows per pass
constexpr int kTcSlots = 8;         // tensor-memory slots of kTcN columns
constexpr int kTcCols = 256;        // columns allocated
constexpr int kTcStage = 16384;     // 128 rows x 128 bytes
constexpr int kTcThreads = 320;     // producer, MMA, 8 epilogue warps
constexpr int kTcEpiWarps = 8;
constexpr int kTcMaxK = 4096;

static __device__ int g_err_tc;

q8_status read_wait_errors_tc(int *flags) {
    cudaError_t e = cudaMemcpyFromSymbol(flags, g_err_tc, sizeof(int));
    return e == cudaSuccess ? Q8_OK : Q8_E_CUDA;
}

struct TcParams {
    CUtensorMap tmap;  // weights as a 2-D int8 tensor [rows_total][k]
    const uint16_t *wd;
    int64_t ld_d;
    int64_t mat_stride;
    int k;
    int rows;       // down: output rows of a matrix
    int n_ff;       // up/gate: gate rows of a matrix (0: down mode)
    const int8_t *aq;
    const uint16_t *ad;
    const float *af;
    int a_per_slot;
    int n_used;
    float *out;
    const int32_t *ws;
    int64_t lay_count, lay_offset, lay_big, lay_pairs;
    int stages;
    int off_x, off_dx, off_xchg, off_dw, off_bar;
};

__device__ __forceinline__ void fence_proxy_async_smem() {
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

__device__ __forceinline__ float tc_silu(float z) { return z / (1.0f + expf(-z)); }

__global__ void __launch_bounds__(kTcThreads, 1) tc_kernel(const __grid_constant__ TcParams p) {
    extern __shared__ __align__(1024) unsigned char smem_raw[];
    // the 128-byte-swizzled stages need 1024-byte alignment
    unsigned char *smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
    griddep_launch_dependents();
    griddep_wait();  // the grouping tables and the activations come from earlier kernels
    if ((int)blockIdx.y >= p.ws[WS_N_BIG]) return;  // uniform: before any barrier
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const bool upgate = p.n_ff > 0;
    const int e = p.ws[p.lay_big + blockIdx.y];
    const int cnt = p.ws[p.lay_count + e];
    const int32_t *plist = p.ws + p.lay_pairs + p.ws[p.lay_offset + e];
    const int row0 = blockIdx.x * (upgate ? 64 : 128);
    const int k = p.k, nb = k / QK, nkc = (k + 127) / 128;

    unsigned char *ring = smem;
    int8_t *xs = reinterpret_cast<int8_t *>(smem + p.off_x);
    float *dxs = reinterpret_cast<float *>(smem + p.off_dx);
    float *xchg = reinterpret_cast<float *>(smem + p.off_xchg);
    uint16_t *dws = reinterpret_cast<uint16_t *>(smem + p.off_dw);  // the tile's weight scales
    uint64_t *wfull = reinterpret_cast<uint64_t *>(smem + p.off_bar);
    uint64_t *wempty = wfull + p.stages;
    uint64_t *sfull = wempty + p.stages;
    uint64_t *sempty = sfull + kTcSlots;
    uint64_t *dfull = sempty + kTcSlots;
    uint32_t *s_tmem = reinterpret_cast<uint32_t *>(dfull + 1);

    if (threadIdx.x == 0) {
        for (int s = 0; s < p.stages; ++s) {
            mbar_init(&wfull[s], 1);
            mbar_init(&wempty[s], 1);
        }
        for (int s = 0; s < kTcSlots; ++s) {
            mbar_init(&sfull[s], 1);
            mbar_init(&sempty[s], kTcEpiWarps);
        }
        mbar_init(dfull, 1);
        fence_barrier_init();
    }
    if (warp == 1) {
        tmem_alloc(s_tmem, kTcCols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *s_tmem;

    int kcg = 0;  // k chunks streamed so far (ring position)
    int bg = 0;   // blocks issued / consumed so far (slot position)
    for (int c0 = 0; c0 < cnt; c0 += kTcN) {
        const int n = min(kTcN, cnt - c0);
        const int npad = (n + 15) / 16 * 16;
        const int ngrp = npad / 8;  // 8-row groups
        __syncthreads();  // the previous pass's MMAs and epilogue are done with xs
        // ---- stage the activation rows as Q8_0, no-swizzle K-major core matrices
        auto arow = [&](int j) {
            const int pr = plist[c0 + j];
            return p.a_per_slot ? pr : pr / p.n_used;
        };
        if (p.af) {
            for (int blk = warp; blk < npad * nb; blk += kTcThreads / 32) {
                const int j = blk / nb, b = blk - j * nb;
                const float v = j < n ? p.af[(int64_t)arow(j) * k + b * QK + lane] : 0.0f;
                const float amax = warp_max_all(fabsf(v));
                const float d32 = block_scale(amax);
                const float id = block_inv_scale(d32);
                const int kbyte = b * QK + lane;
                const int c = kbyte >> 4;
                xs[(c * ngrp + (j >> 3)) * 128 + (j & 7) * 16 + (kbyte & 15)] =
                    (int8_t)quantize_one(v, id);
                if (lane == 0) dxs[j * nb + b] = j < n ? scale_value(scale_bits(d32)) : 0.0f;
            }
        } else {
            const int chunks = k / 16;
            for (int i = threadIdx.x; i < npad * chunks; i += kTcThreads) {
                const int j = i / chunks, c = i - j * chunks;
                uint4 v = make_uint4(0, 0, 0, 0);
                if (j < n) v = *reinterpret_cast<const uint4 *>(p.aq + (int64_t)arow(j) * k + c * 16);
                *reinterpret_cast<uint4 *>(xs + (c * ngrp + (j >> 3)) * 128 + (j & 7) * 16) = v;
            }
            for (int i = threadIdx.x; i < npad * nb; i += kTcThreads) {
                const int j = i / nb, b = i - j * nb;
                dxs[i] = j < n ? scale_value(p.ad[(int64_t)arow(j) * nb + b]) : 0.0f;
            }
        }
        fence_proxy_async_smem();  // generic-proxy writes, read by the tensor cores
        __syncthreads();

        if (warp == 0) {
            // ---- producer: the tile's K chunks through the ring
            if (lane == 0) {
                if (c0 == 0) {  // the tile's scales, once: contiguous rows of ld_d halves
                    const int64_t mrow = (int64_t)e * p.mat_stride;
                    if (upgate) {
                        const uint32_t bytes = (uint32_t)(64 * p.ld_d * 2);
                        mbar_arrive_expect_tx(dfull, 2 * bytes);
                        bulk_g2s(dws, p.wd + (mrow + row0) * p.ld_d, bytes, dfull);
                        bulk_g2s(dws + 64 * p.ld_d, p.wd + (mrow + p.n_ff + row0) * p.ld_d, bytes, dfull);
                    } else {
                        const int valid = min(128, p.rows - row0);
                        const uint32_t bytes = (uint32_t)(valid * p.ld_d * 2);
                        mbar_arrive_expect_tx(dfull, bytes);
                        bulk_g2s(dws, p.wd + (mrow + row0) * p.ld_d, bytes, dfull);
                    }
                }
                for (int kc = 0; kc < nkc; ++kc, ++kcg) {
                    const int s = kcg % p.stages, round = kcg / p.stages;
                    if (round > 0) mbar_wait(&wempty[s], (round - 1) & 1, &g_err_tc);
                    mbar_arrive_expect_tx(&wfull[s], kTcStage);
                    unsigned char *dst = ring + (size_t)s * kTcStage;
                    const int64_t mrow = (int64_t)e * p.mat_stride;
                    if (upgate) {
                        tma_load_2d(dst, &p.tmap, kc * 128, (int)(mrow + row0), &wfull[s]);
                        tma_load_2d(dst + kTcStage / 2, &p.tmap, kc * 128,
                                    (int)(mrow + p.n_ff + row0), &wfull[s]);
                    } else {
                        tma_load_2d(dst, &p.tmap, kc * 128, (int)(mrow + row0), &wfull[s]);
                    }
                }
            } else {
                kcg += nkc;
            }
        } else if (warp == 1) {
            // ---- MMA issuer: one MMA per Q8_0 block into its own slot
            const uint32_t idesc = idesc_i8(npad);
            const uint32_t xs_addr = smem_u32(xs);
            const uint32_t lbo = (uint32_t)ngrp * 128;
            for (int b = 0; b < nb; ++b, ++bg) {
                const int kq = kcg + b / 4;
                const int s = kq % p.stages;
                if (lane == 0) {
                    if ((b & 3) == 0) {
                        mbar_wait(&wfull[s], (kq / p.stages) & 1, &g_err_tc);
                        tc_fence_after();
                    }
                    const int slot = bg % kTcSlots, sround = bg / kTcSlots;
                    if (sround > 0) {
                        mbar_wait(&sempty[slot], (sround - 1) & 1, &g_err_tc);
                        tc_fence_after();
                    }
                    const uint32_t a_addr = smem_u32(ring + (size_t)s * kTcStage) + (b & 3) * 32;
                    const uint64_t adesc = smem_desc(a_addr, 16, 1024, 2);
                    const uint64_t bdesc = smem_desc(xs_addr + (uint32_t)(2 * b) * lbo, lbo, 128, 0);
                    mma_i8(tmem + (uint32_t)(slot * kTcN), adesc, bdesc, idesc, 0);
                    tc_commit(&sfull[slot]);
                    if ((b & 3) == 3 || b == nb - 1) tc_commit(&wempty[s]);
                }
                __syncwarp();
            }
            kcg += nkc;
        } else {
            // ---- epilogue: thread = weight row, 16 activation rows per warp
            const int q = warp & 3;            // tensor-memory lane quarter
            const int half = (warp - 2) >> 2;  // activation rows half*16 .. +16
            const int row = q * 32 + lane;     // tile row (lane of tensor memory)
            int64_t grow;                      // weight row in the matrix
            bool row_ok;
            if (upgate) {
                grow = row < 64 ? row0 + row : p.n_ff + row0 + (row - 64);
                row_ok = true;
            } else {
                grow = row0 + row;
                row_ok = grow < p.rows;
            }
            const uint16_t *drow = dws + (size_t)row * p.ld_d;
            const bool active = half * 16 < npad;
            if (c0 == 0) mbar_wait(dfull, 0, &g_err_tc);
            float acc[16];
#pragma unroll
            for (int t = 0; t < 16; ++t) acc[t] = 0.0f;
            // blocks in groups of up to 4 (one K chunk): the MMA thread's
            // commit on the group's last slot covers the group's earlier
            // MMAs too, so one wait and one tensor-memory load round trip
            // serve four blocks
            for (int b = 0; b < nb; b += 4) {
                const int gn = min(4, nb - b);
                const int slot_last = (bg + gn - 1) % kTcSlots;
                mbar_wait(&sfull[slot_last], ((bg + gn - 1) / kTcSlots) & 1, &g_err_tc);
                tc_fence_after();
                uint32_t v[4][16];
                if (active) {
#pragma unroll
                    for (int i = 0; i < 4; ++i)
                        if (i < gn)
                            tmem_ld16(tmem + ((uint32_t)(q * 32) << 16) +
                                          (uint32_t)(((bg + i) % kTcSlots) * kTcN + half * 16),
                                      v[i]);
                    tmem_ld_wait();
                }
                tc_fence_before();
                __syncwarp();
                if (lane == 0)
                    for (int i = 0; i < gn; ++i) mbar_arrive(&sempty[(bg + i) % kTcSlots]);
                if (active) {
#pragma unroll
                    for (int i = 0; i < 4; ++i) {
                        if (i < gn) {
                            const float dw = row_ok ? scale_value(drow[b + i]) : 0.0f;
                            const float *dxb = dxs + (half * 16) * nb + b + i;
#pragma unroll
                            for (int t = 0; t < 16; ++t)
                                acc[t] = fmaf(dw * dxb[t * nb], small_int_to_float((int)v[i][t]),
                                              acc[t]);
                        }
                    }
                }
                bg += gn;
            }
            // ---- outputs
            if (upgate) {
                if (row >= 64 && active) {
#pragma unroll
                    for (int t = 0; t < 16; ++t) xchg[(row - 64) * kTcN + half * 16 + t] = acc[t];
                }
                named_bar_sync(2, kTcEpiWarps * 32);
                if (row < 64 && active) {
#pragma unroll
                    for (int t = 0; t < 16; ++t) {
                        const int tl = half * 16 + t;
                        if (tl < n) {
                            const float u = xchg[row * kTcN + tl];
                            p.out[(int64_t)plist[c0 + tl] * p.n_ff + row0 + row] = tc_silu(acc[t]) * u;
                        }
                    }
                }
            } else if (row_ok && active) {
#pragma unroll
                for (int t = 0; t < 16; ++t) {
                    const int tl = half * 16 + t;
                    if (tl < n) p.out[(int64_t)plist[c0 + tl] * p.rows + grow] = acc[t];
                }
            }
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, kTcCols);
    }
}

// ---------------------------------------------------------------------------
// host side
// ---------------------------------------------------------------------------
static PFN_cuTensorMapEncodeTiled_v12000 g_encode = nullptr;
static std::once_flag g_encode_once;

static q8_status encode_fn(PFN_cuTensorMapEncodeTiled_v12000 *out) {
    std::call_once(g_encode_once, [] {
        void *fn = nullptr;
        cudaDriverEntryPointQueryResult q{};
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            g_encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
    });
    if (!g_encode) Q8_FAIL(Q8_E_CUDA, "tensor-core path: cuTensorMapEncodeTiled unavailable");
    *out = g_encode;
    return Q8_OK;
}

bool tc_eligible(const q8_tensor *W, bool upgate) {
    if (W->k < 128 || W->k > kTcMaxK || W->k % QK) return false;
    if (upgate && (W->rows / 2) % 64 != 0) return false;
    return true;
}

// Launch the tensor-core kernel over the tensor-core expert list of ws.
// upgate: W is the combined gate/up tensor, out = h [P][n_ff]; else W is
// [n_mat][rows][k], out = y [P][rows].
q8_status launch_tc(const q8_tensor *W, bool upgate, const int8_t *aq, const uint16_t *ad,
                    const float *af, int a_per_slot, int64_t n_tok, int32_t n_used, float *out,
                    const int32_t *ws, cudaStream_t s) {
    const int64_t P = n_tok * n_used;
    const int64_t max_big = std::min<int64_t>(W->n_mat, P / kTcMinPairs);
    if (max_big <= 0) return Q8_OK;  // no expert can reach the threshold
    PFN_cuTensorMapEncodeTiled_v12000 enc;
    q8_status st = encode_fn(&enc);
    if (st != Q8_OK) return st;
    const GroupLayout L = group_layout(P, W->n_mat);
    TcParams p{};
    const int64_t rows_total = (W->n_mat - 1) * W->mat_stride + W->rows;
    cuuint64_t dims[2] = {(cuuint64_t)W->k, (cuuint64_t)rows_total};
    cuuint64_t strides[1] = {(cuuint64_t)W->k};
    cuuint32_t box[2] = {128, (cuuint32_t)(upgate ? 64 : 128)};
    cuuint32_t estr[2] = {1, 1};
    CUresult r = enc(&p.tmap, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, (void *)W->qs, dims, strides, box,
                     estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                     CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) Q8_FAIL(Q8_E_CUDA, "tensor-core path: tensor map encode failed (%d)", (int)r);
    p.wd = W->d;
    p.ld_d = W->ld_d;
    p.mat_stride = W->mat_stride;
    p.k = (int)W->k;
    p.rows = (int)W->rows;
    p.n_ff = upgate ? (int)(W->rows / 2) : 0;
    p.aq = aq;
    p.ad = ad;
    p.af = af;
    p.a_per_slot = a_per_slot;
    p.n_used = n_used;
    p.out = out;
    p.ws = ws;
    p.lay_count = L.count;
    p.lay_offset = L.offset;
    p.lay_big = L.list_big;
    p.lay_pairs = L.pairs;
    // shared memory: ring, activations, their scales, the gate/up exchange, barriers
    const int nb = (int)(W->k / QK);
    const int x_bytes = kTcN * (int)W->k;
    const int dx_bytes = ((kTcN * nb * 4 + 127) / 128) * 128;
    const int xchg_bytes = 64 * kTcN * 4;
    const int dw_bytes = ((int)(128 * W->ld_d * 2) + 127) / 128 * 128;
    const int bar_bytes = 2 * (8 + kTcSlots) * 8 + 32;
    const int fixed = x_bytes + dx_bytes + xchg_bytes + dw_bytes + bar_bytes + 1024;
    int stages = (kSmemLimit - fixed) / kTcStage;
    if (stages > 8) stages = 8;
    if (stages < 2) Q8_FAIL(Q8_E_UNSUPPORTED, "tensor-core path: k=%lld too large", (long long)W->k);
    p.stages = stages;
    p.off_x = stages * kTcStage;
    p.off_dx = p.off_x + x_bytes;
    p.off_xchg = p.off_dx + dx_bytes;
    p.off_dw = p.off_xchg + xchg_bytes;
    p.off_bar = p.off_dw + dw_bytes;
    const int smem = p.off_bar + bar_bytes + 1024;  // + alignment slack
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) Q8_FAIL(Q8_E_CUDA, "tensor-core path: no device");
    if (!smem_opted_in((const void *)tc_kernel, dev)) {
        cudaError_t e = cudaFuncSetAttribute(tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             kSmemLimit);
        if (e != cudaSuccess)
            Q8_FAIL(Q8_E_CUDA, "tensor-core path: shared-memory attribute: %s", cudaGetErrorString(e));
        set_smem_opted_in((const void *)tc_kernel, dev);
    }
    const int tiles = upgate ? (int)(W->rows / 2 / 64) : (int)((W->rows + 127) / 128);
    return launch_pdl("tc_kernel", tc_kernel, dim3((unsigned)tiles, (unsigned)max_big),
                      dim3(kTcThreads), (size_t)smem, s, p);
}

}  // namespace q8
