// q8_tc.cu -- the int8 tensor-core (tcgen05) path of the routed matmuls, for
// experts that receive at least kTcMinPairs routed rows: the fused MoE
// up/gate + SwiGLU and the mul_mat_id down projection.  With that many
// activation rows per expert the step is a real (small) dense contraction,
// so it goes to the tensor cores; below that the dp4a streaming kernels serve.
//
// A persistent grid (one CTA per SM) walks work items (expert, pass of up to
// 32 of its rows, 128-row weight tile; up/gate tiles are 64 gate rows and the
// 64 matching up rows) through one ring whose stages hold, per 128-byte K
// chunk (4 Q8_0 blocks): the weight tile's chunk (2-D TMA, 128-byte swizzle)
// and the activation rows' chunk as Q8_0 in the canonical no-swizzle K-major
// core-matrix layout (gathered by two warps from the rows the pair list
// names).  The MMAs' commit frees a stage; the rows' block scales go to a
// ring of their own, freed by the epilogue.  One tcgen05.mma.kind::i8 per
// Q8_0 block (M=128, N=16/32, K=32) lands in its own tensor-memory slot
// (16 slots: the MMAs run up to four chunks ahead of the epilogue), because
// each block has its own pair of scales and the int32 sum cannot run across
// blocks; sixteen epilogue warps read the slots back, scale each block sum by
// d_w (rounded once) and add d_x times that to the fp32 sums in block order.
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
constexpr int kTcSlots = 16;        // tensor-memory slots of kTcN columns
constexpr int kTcGroups = kTcSlots / 4;  // slot groups: one K chunk's 4 blocks each
constexpr int kTcCols = 512;        // columns allocated (all of them: one CTA per SM)
constexpr int kTcA = 16384;         // A part of a stage: 128 rows x 128 bytes (128B swizzle)
constexpr int kTcB = kTcN * 128;    // B part: kTcN rows x 128 bytes (core matrices)
constexpr int kTcStage = 20480;     // kTcA + kTcB
constexpr int kTcDxRing = 8;        // entries of the activation-scale ring, one per K chunk
constexpr int kTcDx = kTcN * 4 * 4; // an entry: the chunk's 4 blocks' scales d_x, fp32 [block][row]
constexpr int kTcDh = kTcN * 4 * 2; // then d_x as copied, fp16 [row][block]
constexpr int kTcDxEntry = kTcDx + kTcDh;
// Block scaling.  A block sum |v| < 2^22 becomes the fp32 value kTcMagic + v
// exactly by an integer add of v to the bits of kTcMagic.  kTcMagic * d_w is
// exact in fp32 (d_w is an fp16 value, 11 significant bits), so
// fma(kTcMagic + v, d_w, -kTcMagic * d_w) is v * d_w rounded once; the
// epilogue then adds d_x times that to the row's sum.
constexpr float kTcMagic = 12582912.0f;  // 1.5 * 2^23
constexpr uint32_t kTcMagicBits = 0x4B400000u;
constexpr int kTcLag = 3;           // chunks a builder keeps in flight before it reports one
constexpr int kTcEpiWarps = 16;
constexpr int kTcCw = kTcN * 4 / kTcEpiWarps;  // activation rows (columns) per epilogue warp
constexpr int kTcBuildWarps = 2;
constexpr int kTcThreads = (2 + kTcEpiWarps + kTcBuildWarps) * 32;  // 640
static_assert(kTcCw == 8 || kTcCw == 16, "epilogue split");
constexpr int kTcMaxK = 4096;
constexpr int kTcXs = kTcN + 1;     // gate/up exchange row stride (floats): rows land in distinct banks
static_assert(kTcA + kTcB == kTcStage && kTcStage % 1024 == 0, "stage layout");

static __device__ int g_err_tc;

q8_status read_wait_errors_tc(int *flags) {
    cudaError_t e = cudaMemcpyFromSymbol(flags, g_err_tc, sizeof(int));
    return e == cudaSuccess ? Q8_OK : Q8_E_CUDA;
}

q8_status clear_wait_errors_tc() {
    const int zero = 0;
    cudaError_t e = cudaMemcpyToSymbol(g_err_tc, &zero, sizeof(int));
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
    int n_dense;  // > 0: one matrix, its rows the n_dense activation rows (ws unused)
    int x_async;  // Q8_0 activations gathered by cp.async (aq 16-byte, ad 4-byte aligned, nb even)
    int stages;
    int off_dx, off_dws, off_xchg, off_bar;
    int dws_bytes;  // one of the two tile-scale buffers
};

__device__ __forceinline__ void fence_proxy_async_smem() {
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

__device__ __forceinline__ float tc_silu(float z) { return z / (1.0f + expf(-z)); }

// A block sum |v| < 2^22 (int32 bits) as the fp32 value kTcMagic + v, exactly.
__device__ __forceinline__ float biased(uint32_t v) {
    return __int_as_float((int)v + (int)kTcMagicBits);
}

// A warp's kTcCw columns of one slot (this thread's lane).
__device__ __forceinline__ void tmem_ld_cols(uint32_t addr, uint32_t (&v)[16]) { tmem_ld16(addr, v); }
__device__ __forceinline__ void tmem_ld_cols(uint32_t addr, uint32_t (&v)[8]) { tmem_ld8(addr, v); }


// The CTA's work items, in order: (expert of the tensor-core list, pass of
// kTcN of its rows, weight tile).  Every role walks the same sequence.
struct TcItem {
    int mi, pass, tile;     // position
    int e, cnt, c0, n, npad;
    const int32_t *plist;   // nullptr: dense, row j is activation row j
    __device__ __forceinline__ int pair(int j) const { return plist ? plist[j] : j; }
};

struct TcWalk {
    const TcParams *p;
    int n_big, n_tiles;
    __device__ __forceinline__ int count(int mi) const {
        return p->n_dense > 0 ? p->n_dense : p->ws[p->lay_count + p->ws[p->lay_big + mi]];
    }
    __device__ __forceinline__ int passes(int mi) const { return (count(mi) + kTcN - 1) / kTcN; }
    __device__ __forceinline__ void fill(TcItem &it) const {
        if (p->n_dense > 0) {
            it.e = 0;
            it.cnt = p->n_dense;
            it.plist = nullptr;
        } else {
            it.e = p->ws[p->lay_big + it.mi];
            it.cnt = p->ws[p->lay_count + it.e];
            it.plist = p->ws + p->lay_pairs + p->ws[p->lay_offset + it.e];
        }
        it.c0 = it.pass * kTcN;
        it.n = min(kTcN, it.cnt - it.c0);
        it.npad = (it.n + 15) / 16 * 16;
    }
    // the item with index i, given first[mi] = the passes of the experts
    // before mi (first[n_big] = all of them): a binary search
    __device__ __forceinline__ TcItem seek(int64_t i, const int *first) const {
        TcItem it{};
        if (i >= (int64_t)first[n_big] * n_tiles) {
            it.mi = n_big;
            return it;
        }
        int lo = 0, hi = n_big;  // first[lo] * n_tiles <= i < first[hi] * n_tiles
        while (hi - lo > 1) {
            const int mid = (lo + hi) >> 1;
            if ((int64_t)first[mid] * n_tiles <= i)
                lo = mid;
            else
                hi = mid;
        }
        it.mi = lo;
        const int64_t r = i - (int64_t)first[lo] * n_tiles;
        it.pass = (int)(r / n_tiles);
        it.tile = (int)(r % n_tiles);
        fill(it);
        return it;
    }
    __device__ __forceinline__ void next(TcItem &it) const {
        if (++it.tile == n_tiles) {
            it.tile = 0;
            if (++it.pass == passes(it.mi)) {
                it.pass = 0;
                ++it.mi;
            }
        }
        if (it.mi < n_big) fill(it);
    }
};

// Persistent: each CTA takes a contiguous run of the work items and streams
// them through one ring, keeping its tensor memory.  Roles:
//  warp 0        A producer: the tile's K chunks by 2-D TMA (128B swizzle),
//                and the tile's weight scales by bulk copy (two buffers);
//  warp 1        tensor-memory owner and MMA issuer: one kind::i8 MMA per
//                Q8_0 block into its own tensor-memory slot;
//  warps 2-17    epilogue: thread = weight row, kTcCw activation rows per warp;
//  warps 18-19   B builders: the chunk's activation rows (gathered through
//                the pair list) as Q8_0 core matrices into the same stage,
//                their scales into the scale ring.
// A stage is freed by the MMA issuer's commit, a scale entry by the epilogue.
__global__ void __launch_bounds__(kTcThreads, 1) tc_kernel(const __grid_constant__ TcParams p) {
    extern __shared__ __align__(1024) unsigned char smem_raw[];
    // the 128-byte-swizzled stages need 1024-byte alignment
    unsigned char *smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
    Q8_TRACE(0);
    griddep_launch_dependents();
    griddep_wait();  // the grouping tables and the activations come from earlier kernels
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const bool upgate = p.n_ff > 0;
    const int k = p.k, nb = k / QK, nkc = (k + 127) / 128;
    TcWalk W{&p, p.n_dense > 0 ? 1 : p.ws[WS_N_BIG], upgate ? p.n_ff / 64 : (p.rows + 127) / 128};
    // The walk: every tensor-core expert's pass count (loaded by all
    // threads at once), then their running sum by warp 0, in the ring's
    // memory before the ring is used (n_big <= 4096 ints).
    int *first = reinterpret_cast<int *>(smem);
    for (int mi = threadIdx.x; mi < W.n_big; mi += blockDim.x) first[mi] = W.passes(mi);
    __syncthreads();
    if (warp == 0) {
        int run = 0;
        for (int base = 0; base < W.n_big; base += 32) {
            const int v = base + lane < W.n_big ? first[base + lane] : 0;
            int inc = v;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const int u = __shfl_up_sync(0xffffffffu, inc, o);
                if (lane >= o) inc += u;
            }
            if (base + lane < W.n_big) first[base + lane] = run + inc - v;
            run += __shfl_sync(0xffffffffu, inc, 31);
        }
        if (lane == 0) first[W.n_big] = run;
    }
    __syncthreads();
    const int64_t total = (int64_t)first[W.n_big] * W.n_tiles;
    const int64_t i0 = total * blockIdx.x / gridDim.x, i1 = total * (blockIdx.x + 1) / gridDim.x;
    TcItem it = W.seek(i0, first);
    __syncthreads();       // the ring's memory is free again
    if (i0 >= i1) return;  // uniform: before any other barrier

    unsigned char *ring = smem;
    float *xchg = reinterpret_cast<float *>(smem + p.off_xchg);
    uint64_t *full = reinterpret_cast<uint64_t *>(smem + p.off_bar);
    uint64_t *empty = full + p.stages;
    uint64_t *sfull = empty + p.stages;
    uint64_t *sempty = sfull + kTcGroups;
    uint64_t *dfull = sempty + kTcGroups;
    uint64_t *dempty = dfull + 2;
    uint64_t *xfull = dempty + 2;
    uint64_t *xempty = xfull + kTcDxRing;
    uint32_t *s_tmem = reinterpret_cast<uint32_t *>(xempty + kTcDxRing);
    auto dx_entry = [&](int e) { return smem + p.off_dx + (size_t)e * kTcDxEntry; };
    auto dws = [&](int d) {
        return reinterpret_cast<uint16_t *>(smem + p.off_dws + (size_t)d * p.dws_bytes);
    };

    if (threadIdx.x == 0) {
        for (int s = 0; s < p.stages; ++s) {
            mbar_init(&full[s], 1 + kTcBuildWarps);
            mbar_init(&empty[s], 1);  // the MMA issuer's commit once the chunk's MMAs are done
        }
        for (int e = 0; e < kTcDxRing; ++e) {
            mbar_init(&xfull[e], kTcBuildWarps);
            mbar_init(&xempty[e], kTcEpiWarps);
        }
        for (int q4 = 0; q4 < kTcGroups; ++q4) {
            mbar_init(&sfull[q4], 1);
            mbar_init(&sempty[q4], kTcEpiWarps);
        }
        for (int d = 0; d < 2; ++d) {
            mbar_init(&dfull[d], 1);
            mbar_init(&dempty[d], kTcEpiWarps);
        }
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

    int g = 0;   // K chunks so far (ring position)
    // asynchronous builders: the chunks whose copies have been reported
    int reported = 0;
    // a builder thread's part of chunk pc has landed: convert its two fp16
    // scales into the scale entry's fp32 [block][row] table, make the stage's
    // shared-memory writes visible to the tensor cores, report the warp's part
    auto report = [&](int pc) {
        const int s = pc % p.stages, e = pc % kTcDxRing;
        unsigned char *dxe = dx_entry(e);
        const int j = (threadIdx.x - (2 + kTcEpiWarps) * 32) >> 1, h = threadIdx.x & 1;
        const uint32_t two = *reinterpret_cast<const uint32_t *>(dxe + kTcDx + j * 8 + h * 4);
        float *dxs = reinterpret_cast<float *>(dxe);
        dxs[(2 * h) * kTcN + j] = scale_value((uint16_t)(two & 0xffffu));
        dxs[(2 * h + 1) * kTcN + j] = scale_value((uint16_t)(two >> 16));
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) {
            mbar_arrive(&full[s]);
            mbar_arrive(&xfull[e]);
        }
    };
    // a builder may write chunk gg once the MMAs of the stage's previous
    // chunk are done and the epilogue has read the scale entry's previous chunk
    auto builder_wait = [&](int gg) {
        if (gg >= p.stages) mbar_wait(&empty[gg % p.stages], (gg / p.stages - 1) & 1, &g_err_tc);
        if (gg >= kTcDxRing)
            mbar_wait(&xempty[gg % kTcDxRing], (gg / kTcDxRing - 1) & 1, &g_err_tc);
    };
    // The ring cursor of the single-thread roles (producer, MMA issuer): the
    // stage of chunk gg, the parity of its phase, and whether the ring has
    // wrapped (before that every stage is free).  Set once per item and
    // advanced per chunk, so no division by the stage count per chunk.
    struct RingCursor {
        int s, stages;
        uint32_t ph;
        bool wrapped;
        __device__ __forceinline__ RingCursor(int gg, int n)
            : s(gg % n), stages(n), ph((uint32_t)(gg / n) & 1u), wrapped(gg >= n) {}
        __device__ __forceinline__ void next() {
            if (++s == stages) {
                s = 0;
                ph ^= 1u;
                wrapped = true;
            }
        }
    };
    for (int64_t ii = 0; ii < i1 - i0; ++ii, W.next(it)) {
        const int d = (int)(ii & 1);
        const int row0 = it.tile * (upgate ? 64 : 128);
        const int64_t mrow = (int64_t)it.e * p.mat_stride;
        if (warp == 0) {
            // ---- A producer
            if (lane == 0) {
                if (ii >= 2) mbar_wait(&dempty[d], (int)((ii / 2 - 1) & 1), &g_err_tc);
                if (upgate) {
                    const uint32_t bytes = (uint32_t)(64 * p.ld_d * 2);
                    mbar_arrive_expect_tx(&dfull[d], 2 * bytes);
                    bulk_g2s(dws(d), p.wd + (mrow + row0) * p.ld_d, bytes, &dfull[d]);
                    bulk_g2s(dws(d) + 64 * p.ld_d, p.wd + (mrow + p.n_ff + row0) * p.ld_d, bytes,
                             &dfull[d]);
                } else {
                    const int valid = min(128, p.rows - row0);
                    const uint32_t bytes = (uint32_t)(valid * p.ld_d * 2);
                    mbar_arrive_expect_tx(&dfull[d], bytes);
                    bulk_g2s(dws(d), p.wd + (mrow + row0) * p.ld_d, bytes, &dfull[d]);
                }
                RingCursor rc(g, p.stages);
                for (int kc = 0; kc < nkc; ++kc, rc.next()) {
                    if (rc.wrapped) mbar_wait(&empty[rc.s], rc.ph ^ 1u, &g_err_tc);
                    Q8_TRACE(15);
                    mbar_arrive_expect_tx(&full[rc.s], kTcA);
                    unsigned char *dst = ring + (size_t)rc.s * kTcStage;
                    if (upgate) {
                        tma_load_2d(dst, &p.tmap, kc * 128, (int)(mrow + row0), &full[rc.s]);
                        tma_load_2d(dst + kTcA / 2, &p.tmap, kc * 128, (int)(mrow + p.n_ff + row0),
                                    &full[rc.s]);
                    } else {
                        tma_load_2d(dst, &p.tmap, kc * 128, (int)(mrow + row0), &full[rc.s]);
                    }
                }
            }
        } else if (warp >= 2 + kTcEpiWarps && p.x_async) {
            // ---- B builders, asynchronous (Q8_0 activations): thread (row j,
            // blocks 2h and 2h+1 of every chunk) copies its two blocks as four
            // 16-byte pieces straight into their core-matrix places and the
            // two fp16 scales into the stage's staging; a chunk is reported
            // kTcLag chunks later, once its copies have landed, so the gathers
            // of several chunks are in flight at once
            const int j = (threadIdx.x - (2 + kTcEpiWarps) * 32) >> 1, h = threadIdx.x & 1;
            const int ngrp = it.npad / 8;
            const int8_t *xrow = nullptr;
            const uint16_t *dxrow = nullptr;
            if (j < it.n) {
                const int pr = it.pair(it.c0 + j);
                const int64_t r = p.a_per_slot ? pr : pr / p.n_used;
                xrow = p.aq + r * k;
                dxrow = p.ad + r * nb;
            }

            for (int kc = 0; kc < nkc; ++kc) {
                const int gg = g + kc, s = gg % p.stages;
                builder_wait(gg);
                Q8_TRACE(13);
                unsigned char *bst = ring + (size_t)s * kTcStage + kTcA;
                // nb is even, so both blocks of the pair are present or neither
                if (xrow && 2 * h < nb - kc * 4) {
#pragma unroll
                    for (int c = 4 * h; c < 4 * h + 4; ++c)
                        cp_async16(bst + (c * ngrp + (j >> 3)) * 128 + (j & 7) * 16,
                                   xrow + kc * 128 + c * 16);
                    cp_async4(dx_entry(gg % kTcDxRing) + kTcDx + j * 8 + h * 4,
                              dxrow + kc * 4 + 2 * h);
                }
                cp_async_commit();
                if (gg - reported >= kTcLag) {
                    cp_async_wait<kTcLag>();
                    report(reported++);
                }
            }
        } else if (warp >= 2 + kTcEpiWarps) {
            // ---- B builders: thread per (row, block of the chunk); a
            // thread owns items tid and tid + 64 of every chunk (npad * 4 <= 128)
            const int tid = threadIdx.x - (2 + kTcEpiWarps) * 32;
            const int ngrp = it.npad / 8;
            for (int kc = 0; kc < nkc; ++kc) {
                const int gg = g + kc, s = gg % p.stages;
                builder_wait(gg);
                unsigned char *bst = ring + (size_t)s * kTcStage + kTcA;
                float *dxs = reinterpret_cast<float *>(dx_entry(gg % kTcDxRing));
                for (int idx = tid; idx < it.npad * 4; idx += kTcBuildWarps * 32) {
                    const int j = idx >> 2, b4 = idx & 3;
                    const int kb = kc * 4 + b4;
                    uint4 lo = make_uint4(0, 0, 0, 0), hi = lo;
                    float dx = 0.0f;
                    if (j < it.n && kb < nb) {
                        const int pr = it.pair(it.c0 + j);
                        const int64_t r = p.a_per_slot ? pr : pr / p.n_used;
                        if (p.af) {
                            const float4 *src =
                                reinterpret_cast<const float4 *>(p.af + r * k + kb * QK);
                            float v[32];
#pragma unroll
                            for (int i = 0; i < 8; ++i) {
                                const float4 f = src[i];
                                v[4 * i] = f.x;
                                v[4 * i + 1] = f.y;
                                v[4 * i + 2] = f.z;
                                v[4 * i + 3] = f.w;
                            }
                            uint32_t q[8];
                            const float d32 = quantize_block_thread(v, q);
                            lo = make_uint4(q[0], q[1], q[2], q[3]);
                            hi = make_uint4(q[4], q[5], q[6], q[7]);
                            dx = scale_value(scale_bits(d32));
                        } else {
                            const uint4 *src = reinterpret_cast<const uint4 *>(p.aq + r * k + kb * QK);
                            lo = src[0];
                            hi = src[1];
                            dx = scale_value(p.ad[r * nb + kb]);
                        }
                    }
                    // core matrix (16-byte column c, 8-row group j/8)
                    const int c = 2 * b4;
                    *reinterpret_cast<uint4 *>(bst + (c * ngrp + (j >> 3)) * 128 + (j & 7) * 16) = lo;
                    *reinterpret_cast<uint4 *>(bst + ((c + 1) * ngrp + (j >> 3)) * 128 + (j & 7) * 16) = hi;
                    dxs[b4 * kTcN + j] = dx;  // [block][row]: a warp's rows are contiguous
                }
                fence_proxy_async_smem();  // generic-proxy writes, read by the tensor cores
                __syncwarp();
                if (lane == 0) {
                    mbar_arrive(&full[s]);
                    mbar_arrive(&xfull[gg % kTcDxRing]);
                }
            }
        } else if (warp == 1) {
            // ---- MMA issuer
            if (lane == 0) {
                // one thread issues everything, so the per-chunk work is kept
                // small: one wait for the stage, one for the chunk's slot group,
                // descriptors advanced by adds, two commits
                const uint32_t idesc = idesc_i8(it.npad);
                const uint32_t lbo = (uint32_t)(it.npad / 8) * 128;
                const uint64_t bstep = (uint64_t)((2 * lbo) >> 4);  // next block: 2 core-matrix columns
                // stage 0's descriptors; stage s adds s * kTcStage / 16 to the
                // address field (the ring lies below 256 KB: no carry out of it)
                const uint32_t ring0 = smem_u32(ring);
                const uint64_t adesc0 = smem_desc(ring0, 16, 1024, 2);
                const uint64_t bdesc0 = smem_desc(ring0 + kTcA, lbo, 128, 0);
                RingCursor rc(g, p.stages);
                for (int kc = 0; kc < nkc; ++kc, rc.next()) {
                    const int gg = g + kc, grp = gg & (kTcGroups - 1);
                    mbar_wait(&full[rc.s], rc.ph, &g_err_tc);
                    Q8_TRACE(9);
                    if (gg >= kTcGroups) mbar_wait(&sempty[grp], ((gg / kTcGroups) - 1) & 1, &g_err_tc);
                    Q8_TRACE(11);
                    tc_fence_after();
                    const uint64_t soff = (uint64_t)(rc.s * (kTcStage >> 4));
                    uint64_t adesc = adesc0 + soff, bdesc = bdesc0 + soff;
                    uint32_t dt = tmem + (uint32_t)(grp * 4 * kTcN);
                    if (nb - kc * 4 >= 4) {
#pragma unroll
                        for (int b4 = 0; b4 < 4; ++b4) {
                            mma_i8(dt, adesc, bdesc, idesc, 0);
                            adesc += 2;  // 32 bytes along K within the swizzled rows
                            bdesc += bstep;
                            dt += kTcN;
                        }
                    } else {
                        for (int b4 = 0; b4 < nb - kc * 4; ++b4) {
                            mma_i8(dt, adesc, bdesc, idesc, 0);
                            adesc += 2;
                            bdesc += bstep;
                            dt += kTcN;
                        }
                    }
                    tc_commit(&sfull[grp]);   // the chunk's slots hold its block sums
                    tc_commit(&empty[rc.s]);  // the stage is free once these MMAs are done
                    Q8_TRACE(12);
                }
            }
            __syncwarp();
        } else {
            // ---- epilogue
            const int q = warp & 3;            // tensor-memory lane quarter
            const int part = (warp - 2) >> 2;  // activation rows part*kTcCw .. +kTcCw
            const int row = q * 32 + lane;     // tile row (lane of tensor memory)
            int64_t grow;
            bool row_ok;
            if (upgate) {
                grow = row < 64 ? row0 + row : p.n_ff + row0 + (row - 64);
                row_ok = true;
            } else {
                grow = row0 + row;
                row_ok = grow < p.rows;
            }
            // a warp whose columns all lie past the pass's rows (the MMA's N is
            // padded to 16 or 32) reads and scales nothing (skipping the columns
            // past the rows inside a warp's part too measured slower)
            const bool active = part * kTcCw < it.n;
            mbar_wait(&dfull[d], (int)((ii / 2) & 1), &g_err_tc);
            const uint16_t *drow = dws(d) + (size_t)row * p.ld_d;
            float acc[kTcCw];  // the warp's kTcCw activation rows of this thread's weight row
#pragma unroll
            for (int t = 0; t < kTcCw; ++t) acc[t] = 0.0f;
            for (int kc = 0; kc < nkc; ++kc) {
                const int gg = g + kc, grp = gg % kTcGroups;
                const int gn = min(4, nb - kc * 4);
                const int e = gg % kTcDxRing;
                mbar_wait(&xfull[e], (gg / kTcDxRing) & 1, &g_err_tc);
                Q8_TRACE(6);
                const float *dxs = reinterpret_cast<const float *>(dx_entry(e));
                mbar_wait(&sfull[grp], (gg / kTcGroups) & 1, &g_err_tc);
                Q8_TRACE(7);
                tc_fence_after();
                uint32_t v[4][kTcCw];
                if (active) {
                    const uint32_t ta = tmem + ((uint32_t)(q * 32) << 16) +
                                        (uint32_t)(grp * 4 * kTcN + part * kTcCw);
#pragma unroll
                    for (int i = 0; i < 4; ++i) {
                        if (i < gn) tmem_ld_cols(ta + (uint32_t)(i * kTcN), v[i]);
                    }
                    tmem_ld_wait();
                }
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&sempty[grp]);
                if (active) {
                    // the row's 4 weight scales of the chunk in one 8-byte load (ld_d is a
                    // multiple of 8, so the 4 stay inside the row's padded scales)
                    const uint2 dw4 = *reinterpret_cast<const uint2 *>(drow + kc * 4);
                    const uint16_t dwh[4] = {(uint16_t)(dw4.x & 0xffffu), (uint16_t)(dw4.x >> 16),
                                             (uint16_t)(dw4.y & 0xffffu), (uint16_t)(dw4.y >> 16)};
#pragma unroll
                    for (int i = 0; i < 4; ++i) {
                        if (i < gn) {
                            const float dw = row_ok ? scale_value(dwh[i]) : 0.0f;
                            const float dm = -kTcMagic * dw;  // exact
                            // the block's kTcCw activation scales: 16-byte loads;
                            // acc[t] = fma(dx[t], round(v[t] * dw), acc[t]) (scalar fma:
                            // the packed f32x2 form measured 3% slower here; biasing v in
                            // tensor memory, rewritten after every read, 5% slower than
                            // the integer add)
                            const float4 *dx4 =
                                reinterpret_cast<const float4 *>(dxs + i * kTcN + part * kTcCw);
#pragma unroll
                            for (int q4 = 0; q4 < kTcCw / 4; ++q4) {
                                const float4 f = dx4[q4];
                                const int t = 4 * q4;
                                acc[t] = fmaf(f.x, fmaf(biased(v[i][t]), dw, dm), acc[t]);
                                acc[t + 1] = fmaf(f.y, fmaf(biased(v[i][t + 1]), dw, dm), acc[t + 1]);
                                acc[t + 2] = fmaf(f.z, fmaf(biased(v[i][t + 2]), dw, dm), acc[t + 2]);
                                acc[t + 3] = fmaf(f.w, fmaf(biased(v[i][t + 3]), dw, dm), acc[t + 3]);
                            }
                        }
                    }
                }
                Q8_TRACE(8);
                __syncwarp();
                if (lane == 0) mbar_arrive(&xempty[e]);
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(&dempty[d]);
            // ---- outputs
            if (upgate) {
                if (row >= 64 && active) {
#pragma unroll
                    for (int t = 0; t < kTcCw; ++t) xchg[(row - 64) * kTcXs + part * kTcCw + t] = acc[t];
                }
                named_bar_sync(2, kTcEpiWarps * 32);
                if (row < 64 && active) {
#pragma unroll
                    for (int t = 0; t < kTcCw; ++t) {
                        const int tl = part * kTcCw + t;
                        if (tl < it.n) {
                            const float u = xchg[row * kTcXs + tl];
                            p.out[(int64_t)it.pair(it.c0 + tl) * p.n_ff + row0 + row] =
                                tc_silu(acc[t]) * u;
                        }
                    }
                }
                named_bar_sync(2, kTcEpiWarps * 32);  // xchg is free for the next item
                Q8_TRACE(10);
            } else if (row_ok && active) {
#pragma unroll
                for (int t = 0; t < kTcCw; ++t) {
                    const int tl = part * kTcCw + t;
                    if (tl < it.n) p.out[(int64_t)it.pair(it.c0 + tl) * p.rows + grow] = acc[t];
                }
            }
        }
        g += nkc;
    }
    if (warp >= 2 + kTcEpiWarps && p.x_async) {
        cp_async_wait<0>();
        while (reported < g) report(reported++);
    }
    // the last stage commit lands before the CTA's shared memory is released
    if (warp == 1 && lane == 0)
        mbar_wait(&empty[(g - 1) % p.stages], ((g - 1) / p.stages) & 1, &g_err_tc);
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
    const bool dense = ws == nullptr;  // one matrix; its rows are the n_tok activation rows
    const int64_t max_big = dense ? 1 : std::min<int64_t>(W->n_mat, P / kTcMinPairs);
    if (max_big <= 0) return Q8_OK;  // no expert can reach the threshold
    if (af && !aligned16(af))
        Q8_FAIL(Q8_E_ALIGN, "tensor-core path: fp32 activations must be 16-byte aligned");
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
    p.n_dense = dense ? (int)n_tok : 0;
    // the gathers go by cp.async when their 16- and 4-byte pieces are aligned
    p.x_async = !af && aq && ad && W->k % 64 == 0 && aligned16(aq) &&
                (reinterpret_cast<uintptr_t>(ad) & 3u) == 0;
    // shared memory: the ring (A, B and the activation scales per stage),
    // two tile-scale buffers, the gate/up exchange, the barriers
    const int xchg_bytes = (64 * kTcXs * 4 + 127) / 128 * 128;
    const int dws_bytes = ((int)(128 * W->ld_d * 2) + 127) / 128 * 128;
    const int bar_bytes = ((2 * 8 + 2 * kTcGroups + 4 + 2 * kTcDxRing) * 8 + 16 + 127) / 128 * 128;
    const int dx_bytes = kTcDxRing * kTcDxEntry;
    const int fixed = dx_bytes + 2 * dws_bytes + xchg_bytes + bar_bytes + 1024;
    int stages = (kSmemLimit - fixed) / kTcStage;
    if (stages > 8) stages = 8;
    if (stages < 3) Q8_FAIL(Q8_E_UNSUPPORTED, "tensor-core path: k=%lld too large", (long long)W->k);
    if (stages <= kTcLag) p.x_async = 0;  // a builder's lag must stay below the ring depth
    // the walk's running sums sit in the ring's memory at the start
    if ((max_big + 1) * 4 > (int64_t)stages * kTcStage)
        Q8_FAIL(Q8_E_UNSUPPORTED, "tensor-core path: %lld experts", (long long)max_big);
    p.stages = stages;
    p.dws_bytes = dws_bytes;
    p.off_dx = stages * kTcStage;
    p.off_dws = p.off_dx + dx_bytes;
    p.off_xchg = p.off_dws + 2 * dws_bytes;
    p.off_bar = p.off_xchg + xchg_bytes;
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
    // persistent: one CTA per SM (at most one per work item); each CTA finds
    // its run of items from the grouping tables
    const int64_t tiles = upgate ? W->rows / 2 / 64 : (W->rows + 127) / 128;
    const int64_t max_items = tiles * max_big * ((P + kTcN - 1) / kTcN);
    const int grid = (int)std::max<int64_t>(1, std::min<int64_t>(num_sms(), max_items));
    return launch_pdl("tc_kernel", tc_kernel, dim3((unsigned)grid), dim3(kTcThreads), (size_t)smem,
                      s, p);
}

}  // namespace q8
