// q8_stream.cuh -- the weight-streaming engine shared by every Q8_0 matmul
// kernel of libq8 (GEMV, batched GEMV, mul_mat_id, fused up/gate + SwiGLU).
//
// One persistent CTA per SM: warp 8 is the producer, warps 0-7 consume.
//  * The work is a list of weight tiles: nr consecutive rows of one matrix
//    (or nr/2 gate rows and the nr/2 matching up rows), nr fixed by the row
//    length k.  A CTA takes a contiguous run of tiles.
//  * The producer's elected lane streams each tile's quants and scales into a
//    ring of shared-memory stages with 1-D bulk copies (cp.async.bulk, no
//    multicast), several tiles ahead; a stage is refilled once the 8 consumer
//    warps have released it (mbarrier "empty"), and consumers learn that a
//    stage is full from its transaction-count mbarrier ("full").
//  * Consumers stage the activation rows of the tile's matrix in shared memory
//    (Q8_0 rows copied, or fp32 rows quantized on the way in) when the matrix
//    changes, compute the exact int32 block dots with dp4a, scale by
//    d_w * d_x in fp32, reduce each row with a fixed shuffle tree and hand
//    the row sums to the kernel's epilogue through a double-buffered
//    shared array.
//  * Lane mapping: lane l of a warp takes block base + l of its rows (two
//    16-byte shared loads per row and activation row, 8 dp4a per block dot,
//    an exact int32).  The order of every floating-point sum depends only on
//    k, so a row gives bitwise the same result in every kernel.
//  * Programmatic dependent launch: weights never depend on earlier kernels,
//    so a dense producer starts streaming at once; everything that reads
//    activations or routing tables first waits for the preceding grid.
#pragma once

#include <algorithm>
#include <type_traits>

#include "q8_device.cuh"
#include "q8_internal.h"
#include "q8_ptx.cuh"

namespace q8 {

constexpr int kCW = 8;                  // consumer warps
constexpr int kCT = kCW * 32;           // consumer threads
constexpr int kThreadsStream = kCT + 32;
constexpr int kMaxTileQs = 32768;       // quant bytes of one tile at most (nr * k)
constexpr int kMaxStages = 8;
constexpr int kSmemLimit = 227 * 1024;
constexpr int kBarConsumers = 1;        // named barrier of the consumer warps
constexpr int kMaxXRows = 16;           // activation rows staged at once (at most)

// Tile geometry: rows per tile, warps per row (the row's blocks are split
// into wpr segments, one per warp), rows per warp (kCW * rpw / wpr == nr).
// A warp takes rpw rows at once, so each activation block it loads from
// shared memory serves rpw weight rows.  Up to k = 4096 a warp owns whole
// rows (wpr = 1): its sums are final and need no exchange between warps.
// The order of a row's floating-point sum depends on wpr and k only, and wpr
// is a function of k, so every kernel sums a row the same way.
struct Geo {
    int nr, wpr, rpw;
};
__host__ __device__ inline int wpr_for_k(int k) { return k <= 4096 ? 1 : 8; }
// Plain row tiles (at most 32 KB of quants).  nt: activation rows per pass
// of the kernel; at 8 a warp takes 4 rows (k <= 768) so that its rpw * nt
// sums stay within one reduce-scatter (the sum order of a row is the same).
__host__ __device__ inline Geo geo_for_k(int k, int nt = 1) {
    if (k <= 768) return nt >= 8 ? Geo{32, 1, 4} : Geo{40, 1, 5};
    if (k <= 1024) return {32, 1, 4};
    if (k <= 2048) return {16, 1, 2};
    if (k <= 4096) return {8, 1, 1};
    if (k <= 8192) return {4, 8, 4};
    return {2, 8, 2};
}
// Gate/up tiles: nr/2 gate rows and the nr/2 matching up rows; nr/2 divides
// 32.  With whole rows per warp, warp w owns gate rows w*rpw/2 .. and the
// matching up rows, so it forms h itself.
__host__ __device__ inline Geo geo_pair_for_k(int k) {
    if (k <= 1024) return {32, 1, 4};
    if (k <= 4096) return {16, 1, 2};
    return geo_for_k(k);
}

__host__ inline int round128(int v) { return (v + 127) / 128 * 128; }

// Quant and scale bytes of a full tile.
__host__ inline void tile_bytes(const Geo &g, int k, int64_t ld_d, int *qs, int *d) {
    *qs = g.nr * k;
    *d = (int)(g.nr * ld_d * 2);
}

// Partial-sum buffer stride (floats) of one of its two halves.
constexpr int kPartRows = 40;

// Shared-memory plan of one launch (offsets in bytes from the dynamic base).
struct Plan {
    int stages;
    int stage_qs;     // bytes of quants per stage (the scales follow)
    int stage_bytes;  // bytes per stage
    int xmax;       // activation rows the stage holds
    int max_nb;     // blocks per activation row the stage is sized for
    int off_full, off_empty, off_ring, off_xq, off_xd, off_part, off_tab;
    int tab_words;  // routing tables built in shared memory (0: none)
    int bytes;
    int ctas;       // CTAs per SM the plan is sized for
    // fp32 activation rows the producer copies ahead into the raw slot
    // (0: the consumers load them from global memory themselves)
    int raw_rows;
    int off_xfull, off_xempty, off_raw;
};

// Bytes of the raw activation slot at most (fp32 rows copied by the producer).
constexpr int kRawSlotBytes = 16 * 1024;

__host__ inline int plan_part_floats(int nt) { return 2 * kPartRows * nt; }

// CTAs per SM of a streaming kernel: two for one or two activation rows per
// pass (the second CTA hides the first one's barrier and dependency stalls),
// one otherwise (register use).
__host__ __device__ constexpr int ctas_per_sm(int nt) { return nt <= 2 ? 2 : 1; }
// Shared memory one CTA may use (the SM has 228 KB; 1 KB per CTA is reserved).
__host__ inline int smem_budget(int ctas) { return ctas == 2 ? (228 * 1024) / 2 - 1024 : kSmemLimit; }

// tile_qs / tile_d: the largest tile's quant and scale bytes; xrows:
// activation rows wanted in shared memory at once; tab_words: int32 words of
// routing tables to build in shared memory.  As many stages as fit.
__host__ inline bool make_plan_ctas(int tile_qs, int tile_d, int max_k, int xrows, int nt,
                                    int ctas, Plan *out, int tab_words, bool raw) {
    const int budget = smem_budget(ctas);
    const int tab_bytes = ((tab_words * 4 + 15) / 16) * 16;
    const int stage_qs = round128(tile_qs);
    const int stage_bytes = stage_qs + round128(tile_d);
    Plan p{};
    p.max_nb = max_k / QK;
    int xmax = xrows < kMaxXRows ? xrows : kMaxXRows;
    if (xmax < nt) xmax = nt;
    for (;; xmax -= nt) {
        const int x_bytes = xmax * max_k + ((xmax * p.max_nb * 4 + 15) / 16) * 16;
        const int part_bytes = plan_part_floats(nt) * 4;
        const int raw_rows = raw ? std::min(xmax, kRawSlotBytes / (4 * max_k)) : 0;
        const int raw_bytes = raw_rows * 4 * max_k;
        const int fixed = 256 + x_bytes + part_bytes + tab_bytes + raw_bytes;
        int stages = (budget - fixed) / stage_bytes;
        if (stages > kMaxStages) stages = kMaxStages;
        if (stages >= 2 || xmax <= nt) {
            if (stages < 2) return false;
            p.stages = stages;
            p.stage_qs = stage_qs;
            p.stage_bytes = stage_bytes;
            p.xmax = xmax;
            p.off_full = 0;
            p.off_empty = kMaxStages * 8;
            p.off_xfull = 2 * kMaxStages * 8;
            p.off_xempty = p.off_xfull + 8;
            p.off_ring = 256;
            p.off_xq = p.off_ring + stages * stage_bytes;
            p.off_xd = p.off_xq + xmax * max_k;
            p.off_part = p.off_xd + ((xmax * p.max_nb * 4 + 15) / 16) * 16;
            p.off_tab = p.off_part + part_bytes;
            p.tab_words = tab_words;
            p.raw_rows = raw_rows;
            p.off_raw = p.off_tab + tab_bytes;
            p.bytes = p.off_raw + raw_bytes;
            p.ctas = ctas;
            *out = p;
            return true;
        }
    }
}

// Two CTAs per SM where the kernel allows it and each still gets three ring
// stages (or two of 44 KB and more); else one CTA per SM with the whole
// shared memory.  raw: fp32
// activations that the producer may copy ahead (a raw slot is reserved when
// one row of max_k floats fits kRawSlotBytes and the ring keeps its stages).
__host__ inline bool make_plan(int tile_qs, int tile_d, int max_k, int xrows, int nt, Plan *out,
                               int tab_words = 0, bool raw = false) {
    raw = raw && 4 * max_k <= kRawSlotBytes;
    for (int use_raw = raw ? 1 : 0; use_raw >= 0; --use_raw) {
        if (ctas_per_sm(nt) == 2 &&
            make_plan_ctas(tile_qs, tile_d, max_k, xrows, nt, 2, out, tab_words, use_raw) &&
            (out->stages >= 3 || out->stages * out->stage_bytes >= 88 * 1024))
            return true;
    }
    for (int use_raw = raw ? 1 : 0; use_raw >= 0; --use_raw)
        if (make_plan_ctas(tile_qs, tile_d, max_k, xrows, nt, 1, out, tab_words, use_raw) &&
            (out->stages >= 3 || !use_raw))
            return true;
    return false;
}

// Contiguous run of tiles for this CTA.
__device__ __forceinline__ void my_tiles(int64_t total, int64_t *b, int64_t *e) {
    *b = total * blockIdx.x / gridDim.x;
    *e = total * (blockIdx.x + 1) / gridDim.x;
}

// A tile's weight source: up to two row spans of one matrix.  Span 1 (if any)
// lands at shared row row_off1.
struct TileSrc {
    const int8_t *q0;
    const uint16_t *d0;
    int rows0;
    const int8_t *q1;
    const uint16_t *d1;
    int rows1;
    int row_off1;
    int k;
    int ld_d;
};

struct Ring {
    uint64_t *full;
    uint64_t *empty;
    unsigned char *base;
    int stages;
    int stage_bytes;
    int stage_qs;
    // raw activation slot: fp32 rows copied by the producer (raw_rows == 0: none)
    uint64_t *xfull;
    uint64_t *xempty;
    float *raw;
    int raw_rows;
    __device__ __forceinline__ int8_t *qs(int s) const {
        return reinterpret_cast<int8_t *>(base + (size_t)s * stage_bytes);
    }
    __device__ __forceinline__ uint16_t *d(int s) const {
        return reinterpret_cast<uint16_t *>(base + (size_t)s * stage_bytes + stage_qs);
    }
};

__device__ __forceinline__ Ring ring_init(unsigned char *smem, const Plan &pl) {
    Ring R;
    R.full = reinterpret_cast<uint64_t *>(smem + pl.off_full);
    R.empty = reinterpret_cast<uint64_t *>(smem + pl.off_empty);
    R.base = smem + pl.off_ring;
    R.stages = pl.stages;
    R.stage_bytes = pl.stage_bytes;
    R.stage_qs = pl.stage_qs;
    R.xfull = reinterpret_cast<uint64_t *>(smem + pl.off_xfull);
    R.xempty = reinterpret_cast<uint64_t *>(smem + pl.off_xempty);
    R.raw = reinterpret_cast<float *>(smem + pl.off_raw);
    R.raw_rows = pl.raw_rows;
    if (threadIdx.x == 0) {
        for (int s = 0; s < pl.stages; ++s) {
            mbar_init(&R.full[s], 1);
            mbar_init(&R.empty[s], kCW);
        }
        mbar_init(R.xfull, 1);
        mbar_init(R.xempty, kCW);
        fence_barrier_init();
    }
    __syncthreads();
    return R;
}

// Activation jobs: the consumers stage a new set of activation rows whenever
// the (key, group) of the rows a pass needs changes.  When the rows are fp32
// and fit the raw slot, the producer copies them into the slot in stream
// order (right before the first weight tile that needs them), so they arrive
// behind the weights already in flight instead of being loaded by the
// consumers behind the whole stream; the consumers quantize them from shared
// memory and release the slot.
struct XJobs {
    int key = -1, grp = -1;  // the job last seen
    int n = 0;               // jobs that went through the raw slot
    // true when (key, grp) starts a new job
    __device__ __forceinline__ bool next(int k, int g) {
        if (k == key && g == grp) return false;
        key = k;
        grp = g;
        return true;
    }
};

// Producer side of a job of nx fp32 rows of k floats, row j at row(j).
// bulk copies of 16-byte aligned rows; no L2 eviction hint (other CTAs read
// the same rows).
template <class RowFn>
__device__ __forceinline__ void produce_job(const Ring &R, XJobs &J, int key, int grp, int nx,
                                            int k, RowFn row, int *err) {
    if (!J.next(key, grp) || nx > R.raw_rows) return;
    if (J.n > 0) mbar_wait(R.xempty, (J.n - 1) & 1, err);
    const uint32_t bytes = (uint32_t)k * 4;
    mbar_arrive_expect_tx(R.xfull, bytes * (uint32_t)nx);
    for (int j = 0; j < nx; ++j) bulk_g2s_keep(R.raw + (size_t)j * k, row(j), bytes, R.xfull);
    ++J.n;
}

// No activation jobs (activations staged by the consumers).
struct NoJobs {
    __device__ __forceinline__ void operator()(int64_t, int) const {}
};

// Producer (one lane): stream tiles [tb, te) through the ring.  src(t) gives a
// tile's spans; jobs(t, when) issues the activation jobs of tile t: when == 0
// before its weights (the job of its first group), when == 1 after them (the
// jobs of its other groups).  Ends after the last copies have landed.
// gated: the activations may be written by the preceding grid and this
// thread has not waited for it yet.  The weights do not depend on that grid,
// so the first tile is issued at once; the producer then waits for the grid,
// issues that tile's jobs (its consumers wait for them) and goes on in stream
// order.
template <class SrcFn, class JobFn = NoJobs>
__device__ __forceinline__ void produce(const Ring &R, int64_t tb, int64_t te, SrcFn src,
                                        int *err, JobFn jobs = JobFn{}, bool gated = false) {
    int it = 0;
    Q8_TRACE(20);
    const int64_t pre = gated ? min(te, tb + 1) : tb;
    for (int64_t t = tb; t < te; ++t, ++it) {
        const int s = it % R.stages;
        const int round = it / R.stages;
        if (t == pre && gated) {
            griddep_wait();
            for (int64_t j = tb; j < pre; ++j) {
                jobs(j, 0);
                jobs(j, 1);
            }
        }
        if (t >= pre) jobs(t, 0);
        if (round > 0) mbar_wait(&R.empty[s], (round - 1) & 1, err);
        Q8_TRACE(21);
        const TileSrc ts = src(t);
        const int k = ts.k;
        const int ld_d = ts.ld_d;
        const uint32_t qb0 = (uint32_t)ts.rows0 * k, qb1 = (uint32_t)ts.rows1 * k;
        const uint32_t db0 = (uint32_t)(ts.rows0 * ld_d * 2), db1 = (uint32_t)(ts.rows1 * ld_d * 2);
        mbar_arrive_expect_tx(&R.full[s], qb0 + qb1 + db0 + db1);
        bulk_g2s(R.qs(s), ts.q0, qb0, &R.full[s]);
        bulk_g2s(R.d(s), ts.d0, db0, &R.full[s]);
        if (ts.rows1 > 0) {
            bulk_g2s(R.qs(s) + (size_t)ts.row_off1 * k, ts.q1, qb1, &R.full[s]);
            bulk_g2s(R.d(s) + (size_t)ts.row_off1 * ld_d, ts.d1, db1, &R.full[s]);
        }
        if (t >= pre) jobs(t, 1);
    }
    if (gated && pre == te) {  // every tile went out before the wait
        griddep_wait();
        for (int64_t j = tb; j < te; ++j) {
            jobs(j, 0);
            jobs(j, 1);
        }
    }
    Q8_TRACE(22);
    const int first = it > R.stages ? it - R.stages : 0;
    for (int j = first; j < it; ++j) mbar_wait(&R.full[j % R.stages], (j / R.stages) & 1, err);
    Q8_TRACE(23);
}

// ---------------------------------------------------------------------------
// Expert grouping inside one CTA (all threads), for small batches: the tables
// of GroupLayout L (counts, offsets, the ascending list of experts with
// pairs, the pairs sorted by expert then by pair index) are built in shared
// memory `tab` from ids [n_tok][n_used].  The same stable counting sort as
// the grouping kernel; every CTA builds its own copy.  Routing-id errors are
// recorded in tab[WS_ERR] and, by CTA 0, in *err_out (if given).  The
// tensor-core list is not used here; its words serve as the scatter cursors.
// ---------------------------------------------------------------------------
// The grouping of at most 32 pairs by one warp (all its lanes), with no CTA
// barrier: each lane is a pair, ranks come from shuffles.  Same tables as
// cta_group.
__device__ __forceinline__ void group_small_warp(const int32_t *__restrict__ ids, int n_tok,
                                                 int n_used, int n_mat, const GroupLayout &L,
                                                 int32_t *tab, int32_t *err_out) {
    const int P = n_tok * n_used;
    const int lane = threadIdx.x & 31;
    const bool live = lane < P;
    const int e = live ? ids[lane] : -1;
    const bool valid = live && e >= 0 && e < n_mat;
    int err = (live && !valid) ? ERR_ID_RANGE : 0;
    const unsigned lt = (1u << lane) - 1u;
    // the lanes naming the same expert (invalid lanes match nobody)
    const unsigned peers = __match_any_sync(0xffffffffu, valid ? e : n_mat + lane);
    const bool first = valid && (peers & lt) == 0u;
    const unsigned vb = __ballot_sync(0xffffffffu, valid);
    const unsigned firsts = __ballot_sync(0xffffffffu, first);
    // a repeat: an earlier slot of the same token names the same expert
    const int tok0 = live ? (lane / n_used) * n_used : 0;
    const unsigned tok_mask = (unsigned)((((uint64_t)1 << n_used) - 1u) << tok0);
    if (valid && (peers & lt & tok_mask) != 0u) err |= ERR_ID_REPEAT;
    // rank: the valid pairs of smaller experts, then this expert's earlier
    // pairs; dpos: the distinct smaller experts
    int rank = __popc(peers & lt), dpos = 0;
#pragma unroll
    for (int s2 = 0; s2 < 32; ++s2) {
        const int e2 = __shfl_sync(0xffffffffu, e, s2);
        if (e2 < e) {
            rank += (int)((vb >> s2) & 1u);
            dpos += (int)((firsts >> s2) & 1u);
        }
    }
    if (valid) tab[L.pairs + rank] = lane;
    if (first) {
        tab[L.list_small + dpos] = e;
        tab[L.count + e] = __popc(peers);
        tab[L.offset + e] = rank;
    }
#pragma unroll
    for (int o = 16; o >= 1; o >>= 1) err |= __shfl_xor_sync(0xffffffffu, err, o);
    if (lane == 0) {
        tab[WS_ERR] = err;
        tab[WS_N_SMALL] = __popc(firsts);
        tab[WS_N_BIG] = 0;
        tab[WS_N_PAIRS] = P;
        tab[L.offset + n_mat] = __popc(vb);
        if (err_out && blockIdx.x == 0) *err_out = err;
    }
}

__device__ __forceinline__ void cta_group(const int32_t *__restrict__ ids, int n_tok, int n_used,
                                          int n_mat, const GroupLayout &L, int32_t *tab,
                                          int32_t *err_out) {
    const int P = n_tok * n_used;
    if (P <= 32) {
        if (threadIdx.x < 32) group_small_warp(ids, n_tok, n_used, n_mat, L, tab, err_out);
        __syncthreads();
        return;
    }
    int *cnt = tab + L.count;
    int *cursor = tab + L.list_big;
    int *sid = tab + L.pairs;  // the ids, read once; the pair list overwrites them below
    for (int e = threadIdx.x; e < n_mat; e += blockDim.x) cnt[e] = 0;
    for (int p = threadIdx.x; p < P; p += blockDim.x) sid[p] = ids[p];
    if (threadIdx.x == 0) tab[WS_ERR] = 0;
    __syncthreads();
    int err = 0;
    for (int p = threadIdx.x; p < P; p += blockDim.x) {
        const int e = sid[p];
        if (e < 0 || e >= n_mat) {
            err |= ERR_ID_RANGE;
            continue;
        }
        atomicAdd(&cnt[e], 1);
        const int t = p / n_used;
        for (int s2 = t * n_used; s2 < p; ++s2)
            if (sid[s2] == e) err |= ERR_ID_REPEAT;
    }
    if (err) atomicOr(&tab[WS_ERR], err);
    __syncthreads();
    // each thread keeps the ids of the pairs warp 0 will scatter, because the
    // scatter writes the sorted pairs over sid
    
    const int lane = threadIdx.x & 31;
    if (threadIdx.x < 32) {
        int running = 0, n_small = 0;
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
                tab[L.offset + e] = off;
                cursor[e] = off;
            }
            const unsigned bs = __ballot_sync(0xffffffffu, c > 0);
            if (c > 0) tab[L.list_small + n_small + __popc(bs & ((1u << lane) - 1u))] = e;
            n_small += __popc(bs);
            running += __shfl_sync(0xffffffffu, incl, 31);
        }
        if (lane == 0) {
            tab[L.offset + n_mat] = running;
            tab[WS_N_SMALL] = n_small;
            tab[WS_N_BIG] = 0;
            tab[WS_N_PAIRS] = P;
        }
        __syncwarp();
        for (int base = 0; base < P; base += 32) {
            const int p = base + lane;
            const int e = p < P ? ids[p] : -1;  // global (L1/L2 hit): sid is being overwritten
            const bool valid = e >= 0 && e < n_mat;
            const int key = valid ? e : n_mat + lane;
            const unsigned m = __match_any_sync(0xffffffffu, key);
            const int rank = __popc(m & ((1u << lane) - 1u));
            if (valid) tab[L.pairs + cursor[e] + rank] = p;
            __syncwarp();
            if (valid && (__ffs(m) - 1) == lane) cursor[e] += __popc(m);
            __syncwarp();
        }
        if (err_out && blockIdx.x == 0 && lane == 0) *err_out = tab[WS_ERR];
    }
    __syncthreads();
}

// ---------------------------------------------------------------------------
// activation staging (consumer threads only: threadIdx.x < kCT)
// ---------------------------------------------------------------------------
struct XStage {
    int8_t *q;   // [xmax][k]
    float *dx;   // [xmax][nb]
};

// Copy Q8_0 rows arow(j) of aq/ad, j < n, into the stage.  Wide: each
// thread issues the loads of a whole round (up to 4 quant vectors and 4
// scales) before its first store, one memory latency per round of 4 * kCT
// vectors, where a loop of one load and one shared store per step pays one
// per step (the store may alias the next load as far as the compiler
// knows).  Wide is for dense kernels, for the register-pressure reason given
// at stage_f32.
template <bool Wide = false, class RowFn>
__device__ __forceinline__ void stage_q8(const XStage &xs, const int8_t *__restrict__ aq,
                                         const uint16_t *__restrict__ ad, int k, int n,
                                         RowFn arow) {
    const int nb = k / QK;
    const int v_per_row = k / 16;
    if constexpr (Wide) {
        constexpr int kU = 4;
        const int nv = n * v_per_row, nd = n * nb;
        const int tid = (int)threadIdx.x;
        for (int base = 0; base < nv || base < nd; base += kU * kCT) {
            uint4 v[kU];
            uint16_t d[kU];
#pragma unroll
            for (int u = 0; u < kU; ++u) {
                const int i = base + u * kCT + tid;
                if (i < nv) {
                    const int j = i / v_per_row;
                    const int c = i - j * v_per_row;
                    v[u] = *reinterpret_cast<const uint4 *>(aq + (int64_t)arow(j) * k + c * 16);
                }
                if (i < nd) {
                    const int j = i / nb;
                    d[u] = ad[(int64_t)arow(j) * nb + (i - j * nb)];
                }
            }
#pragma unroll
            for (int u = 0; u < kU; ++u) {
                const int i = base + u * kCT + tid;
                if (i < nv) {
                    const int j = i / v_per_row;
                    const int c = i - j * v_per_row;
                    *reinterpret_cast<uint4 *>(xs.q + (size_t)j * k + c * 16) = v[u];
                }
                if (i < nd) xs.dx[i] = scale_value(d[u]);  // row j = i / nb, block i - j * nb
            }
        }
        return;
    }
#pragma unroll 4
    for (int i = threadIdx.x; i < n * v_per_row; i += kCT) {
        const int j = i / v_per_row;
        const int c = i - j * v_per_row;
        const uint4 v = *reinterpret_cast<const uint4 *>(aq + (int64_t)arow(j) * k + c * 16);
        *reinterpret_cast<uint4 *>(xs.q + (size_t)j * k + c * 16) = v;
    }
    for (int i = threadIdx.x; i < n * nb; i += kCT) {
        const int j = i / nb;
        const int b = i - j * nb;
        xs.dx[(size_t)j * nb + b] = scale_value(ad[(int64_t)arow(j) * nb + b]);
    }
}

// Quantize fp32 rows arow(j) of af (16-byte aligned, k floats apart), j < n,
// into the stage with eight threads per 32-block (thread i takes elements
// 4i..4i+3, as in stage_f32_smem8); each thread issues the loads of kWide of
// its blocks before it quantizes any, so a stage costs one memory latency
// per kWide * kCT / 8 blocks (14336 floats: 2) where one warp per block
// with 8 blocks' loads in flight pays one per 8 blocks of a warp (7).
template <class RowFn>
__device__ __forceinline__ void stage_f32_wide(const XStage xs, const float *__restrict__ af,
                                               int k, int n, RowFn arow) {
    const int nb = k / QK;
    const int total = n * nb;
    constexpr int kWide = 8;
    constexpr int ngrp = kCT / 8;
    const int grp = (int)threadIdx.x >> 3, part = (int)threadIdx.x & 7;
    for (int base = 0; base < total; base += kWide * ngrp) {  // the same trip count in every lane
        float4 f[kWide];
#pragma unroll
        for (int r = 0; r < kWide; ++r) {
            const int blk = base + r * ngrp + grp;
            f[r] = make_float4(0.0f, 0.0f, 0.0f, 0.0f);
            if (blk < total) {
                const int j = blk / nb;
                const int b = blk - j * nb;
                f[r] = reinterpret_cast<const float4 *>(af + (int64_t)arow(j) * k + b * QK)[part];
            }
        }
#pragma unroll
        for (int r = 0; r < kWide; ++r) {
            const int blk = base + r * ngrp + grp;
            float amax = fmaxf(fmaxf(fabsf(f[r].x), fabsf(f[r].y)),
                               fmaxf(fabsf(f[r].z), fabsf(f[r].w)));
            amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 1));
            amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 2));
            amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 4));
            if (blk < total) {
                const int j = blk / nb;
                const int b = blk - j * nb;
                const float d32 = block_scale(amax);
                const float id = block_inv_scale(d32);
                const uint32_t w = ((uint32_t)quantize_one(f[r].x, id) & 0xffu) |
                                   (((uint32_t)quantize_one(f[r].y, id) & 0xffu) << 8) |
                                   (((uint32_t)quantize_one(f[r].z, id) & 0xffu) << 16) |
                                   (((uint32_t)quantize_one(f[r].w, id) & 0xffu) << 24);
                *reinterpret_cast<uint32_t *>(xs.q + (size_t)j * k + b * QK + 4 * part) = w;
                if (part == 0) xs.dx[(size_t)j * nb + b] = scale_value(scale_bits(d32));
            }
        }
    }
}

// Quantize fp32 rows arow(j) of af (k floats apart), j < n, into the stage
// by the Q8_0 rule.  Aligned rows: one thread per 32-block when the blocks
// are at most kCT, else (Wide) eight threads per block with many blocks'
// loads in flight per thread.  Otherwise one warp per 32-block, each warp
// first issuing the loads of up to 8 of its blocks.  amax is an exact
// maximum and every code is formed as in quantize_block_thread, so the three
// forms give the same bits.  Wide is for kernels that stage long or many
// rows (dense matmuls): its loads, inlined, raise the register pressure of
// the dot loops, which costs the routed kernels more than it saves them.
template <bool Wide, class RowFn>
__device__ __forceinline__ void stage_f32(const XStage &xs, const float *__restrict__ af, int k,
                                          int n, RowFn arow) {
    constexpr int kBatch = 8;
    const int nb = k / QK;
    const int lane = threadIdx.x & 31;
    const int total = n * nb;
    if (total <= kCT && ((uintptr_t)af & 15u) == 0) {
        // one block per thread: every load of the stage in flight at once
        if ((int)threadIdx.x < total) {
            const int j = threadIdx.x / nb;
            const int b = threadIdx.x - j * nb;
            const float4 *src =
                reinterpret_cast<const float4 *>(af + (int64_t)arow(j) * k + b * QK);
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
            uint4 *dst = reinterpret_cast<uint4 *>(xs.q + (size_t)j * k + b * QK);
            dst[0] = make_uint4(q[0], q[1], q[2], q[3]);
            dst[1] = make_uint4(q[4], q[5], q[6], q[7]);
            xs.dx[(size_t)j * nb + b] = scale_value(scale_bits(d32));
        }
        return;
    }
    if constexpr (Wide) {
        if (((uintptr_t)af & 15u) == 0) {
            stage_f32_wide(xs, af, k, n, arow);
            return;
        }
    }
    for (int b0 = threadIdx.x >> 5; b0 < total; b0 += kCW * kBatch) {
        float v[kBatch];
#pragma unroll
        for (int i = 0; i < kBatch; ++i) {
            const int blk = b0 + i * kCW;
            v[i] = 0.0f;
            if (blk < total) {
                const int j = blk / nb;
                const int b = blk - j * nb;
                v[i] = af[(int64_t)arow(j) * k + b * QK + lane];
            }
        }
#pragma unroll
        for (int i = 0; i < kBatch; ++i) {
            const int blk = b0 + i * kCW;  // warp-uniform
            if (blk < total) {
                const int j = blk / nb;
                const int b = blk - j * nb;
                const float amax = warp_max_all(fabsf(v[i]));
                const float d32 = block_scale(amax);
                const float id = block_inv_scale(d32);
                xs.q[(size_t)j * k + b * QK + lane] = (int8_t)quantize_one(v[i], id);
                if (lane == 0) xs.dx[(size_t)j * nb + b] = scale_value(scale_bits(d32));
            }
        }
    }
}

// Quantize n fp32 rows held in shared memory (row j at src + arow(j) * k)
// into the stage by the Q8_0 rule, eight threads per 32-block: thread i of an
// aligned group of eight takes elements 4i..4i+3, the block's amax comes from
// three xor shuffles inside the group, and each thread quantizes its own four
// values.  Every element goes through the same operations as in the
// one-thread form (amax is an exact maximum), so the bits are the same; the
// dependent chain per thread is a quarter as long.  tid/nthr: this thread's
// index among the nthr threads (whole warps) that share the work.
template <class RowFn>
__device__ __forceinline__ void stage_f32_smem8(const XStage &xs, const float *src, int k, int n,
                                                RowFn arow, int tid, int nthr) {
    const int nb = k / QK;
    const int total = n * nb;
    const int grp = tid >> 3, part = tid & 7;
    const int ngrp = nthr >> 3;
    for (int base = 0; base < total; base += ngrp) {  // the same trip count in every lane
        const int blk = base + grp;
        const bool live = blk < total;
        int j = 0, b = 0;
        float4 f = make_float4(0.0f, 0.0f, 0.0f, 0.0f);
        if (live) {
            j = blk / nb;
            b = blk - j * nb;
            f = reinterpret_cast<const float4 *>(src + (size_t)arow(j) * k + b * QK)[part];
        }
        float amax = fmaxf(fmaxf(fabsf(f.x), fabsf(f.y)), fmaxf(fabsf(f.z), fabsf(f.w)));
        amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 1));
        amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 2));
        amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 4));
        if (live) {
            const float d32 = block_scale(amax);
            const float id = block_inv_scale(d32);
            const uint32_t w = ((uint32_t)quantize_one(f.x, id) & 0xffu) |
                               (((uint32_t)quantize_one(f.y, id) & 0xffu) << 8) |
                               (((uint32_t)quantize_one(f.z, id) & 0xffu) << 16) |
                               (((uint32_t)quantize_one(f.w, id) & 0xffu) << 24);
            *reinterpret_cast<uint32_t *>(xs.q + (size_t)j * k + b * QK + 4 * part) = w;
            if (part == 0) xs.dx[(size_t)j * nb + b] = scale_value(scale_bits(d32));
        }
    }
}

// The same with TPB threads per 32-block (TPB = 2, 4 or 8): fewer rounds of
// the block's scale divisions when the rows are few and the threads many
// (8 rows of 704 take one round of 2 threads per block among 512 threads,
// against three of 8).  amax is exact and every code is formed as in
// quantize_block_thread, so the bits do not depend on TPB.
template <int TPB, class RowFn>
__device__ __forceinline__ void stage_f32_smem_tpb(const XStage &xs, const float *src, int k,
                                                   int n, RowFn arow, int tid, int nthr) {
    static_assert(TPB == 2 || TPB == 4 || TPB == 8, "threads per block");
    constexpr int F4 = 8 / TPB;  // float4s of the block per thread
    const int nb = k / QK;
    const int total = n * nb;
    const int grp = tid / TPB, part = tid % TPB;
    const int ngrp = nthr / TPB;
    for (int base = 0; base < total; base += ngrp) {  // the same trip count in every lane
        const int blk = base + grp;
        const bool live = blk < total;
        int j = 0, b = 0;
        float4 f[F4];
#pragma unroll
        for (int i = 0; i < F4; ++i) f[i] = make_float4(0.0f, 0.0f, 0.0f, 0.0f);
        if (live) {
            j = blk / nb;
            b = blk - j * nb;
            const float4 *p4 = reinterpret_cast<const float4 *>(src + (size_t)arow(j) * k + b * QK);
#pragma unroll
            for (int i = 0; i < F4; ++i) f[i] = p4[part * F4 + i];
        }
        float amax = 0.0f;
#pragma unroll
        for (int i = 0; i < F4; ++i)
            amax = fmaxf(amax, fmaxf(fmaxf(fabsf(f[i].x), fabsf(f[i].y)),
                                     fmaxf(fabsf(f[i].z), fabsf(f[i].w))));
#pragma unroll
        for (int o = 1; o < TPB; o <<= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
        if (live) {
            const float d32 = block_scale(amax);
            const float id = block_inv_scale(d32);
            uint32_t w[F4];
#pragma unroll
            for (int i = 0; i < F4; ++i)
                w[i] = ((uint32_t)quantize_one(f[i].x, id) & 0xffu) |
                       (((uint32_t)quantize_one(f[i].y, id) & 0xffu) << 8) |
                       (((uint32_t)quantize_one(f[i].z, id) & 0xffu) << 16) |
                       (((uint32_t)quantize_one(f[i].w, id) & 0xffu) << 24);
            uint32_t *dst = reinterpret_cast<uint32_t *>(xs.q + (size_t)j * k + b * QK + 4 * F4 * part);
#pragma unroll
            for (int i = 0; i < F4; ++i) dst[i] = w[i];
            if (part == 0) xs.dx[(size_t)j * nb + b] = scale_value(scale_bits(d32));
        }
    }
}

// Quantize the n fp32 rows of the raw slot (row j at raw + j * k) into the
// stage (stage_f32_smem8).  tid/nthr: this thread's index among the nthr
// threads (whole warps) that share the work (default: the consumer threads).
__device__ __forceinline__ void stage_f32_raw(const XStage &xs, const float *raw, int k, int n,
                                              int tid = -1, int nthr = kCT) {
    stage_f32_smem8(xs, raw, k, n, [](int j) { return j; }, tid < 0 ? (int)threadIdx.x : tid,
                    nthr);
}

// Consumer side of an activation job of nx rows (fp32 af, rows arow(j)):
// from the raw slot when the producer copied them, else from global memory.
// The caller synchronizes the consumer warps afterwards.
template <bool Wide = false, class RowFn>
__device__ __forceinline__ void stage_job_f32(const Ring &R, XJobs &J, const XStage &xs,
                                              const float *af, int k, int nx, RowFn arow,
                                              int *err) {
    if (nx <= R.raw_rows) {
        mbar_wait(R.xfull, J.n & 1, err);
        stage_f32_raw(xs, R.raw, k, nx);
        __syncwarp();
        if ((threadIdx.x & 31) == 0) mbar_arrive(R.xempty);
        ++J.n;
    } else {
        stage_f32<Wide>(xs, af, k, nx, arow);
    }
}

// ---------------------------------------------------------------------------
// the dot engine
// ---------------------------------------------------------------------------

// Exact float of an int32 with |v| < 2^22: v + 1.5 * 2^23 is formed in the
// float's bit pattern (ulp 1 in [2^23, 2^24)), then 1.5 * 2^23 is subtracted
// exactly.  Keeps the conversion on the integer and FMA pipes.
__device__ __forceinline__ float small_int_to_float(int v) {
    return __int_as_float(v + 0x4B400000) - 12582912.0f;
}

// acc[r][t] = this lane's part of the sum over the warp's blocks of stage row
// srow(r) with activation row (xrow0 + t), t < n; srow(r) = row0 + r for
// r < split, row1 + (r - split) after.
// Lane l takes block base + l (both 16-byte halves), so each block dot is
// 8 dp4a in one lane; |isum| <= 32 * 128 * 128 < 2^22.
template <int NT, int RPW>
__device__ __forceinline__ void dot_rows(const int8_t *sq, const uint16_t *sd, int k, int ld_d,
                                         int row0, int row1, int split, int seg, int wpr,
                                         const XStage &xs, int xrow0, int n,
                                         float (&acc)[RPW][NT]) {
    const int lane = threadIdx.x & 31;
    const int nb = k / QK;
    // Lanes 4-7 of every quarter warp load the upper 16 bytes of their block
    // first: a quarter warp's first (and second) loads then fall on 8 distinct
    // 16-byte bank groups (no bank conflicts).  The int32 sum of the two
    // halves does not depend on the order.
    const int h0 = ((lane >> 2) & 1) * 16;
    const int h1 = 16 - h0;
#pragma unroll
    for (int r = 0; r < RPW; ++r)
#pragma unroll
        for (int t = 0; t < NT; ++t) acc[r][t] = 0.0f;
    for (int base = seg * 32; base < nb; base += 32 * wpr) {
        const int kb = base + lane;
        if (kb < nb) {
            uint4 w0[RPW], w1[RPW];
            float dw[RPW];
#pragma unroll
            for (int r = 0; r < RPW; ++r) {
                const int srow = r < split ? row0 + r : row1 + (r - split);
                const int8_t *p = sq + (size_t)srow * k + kb * QK;
                w0[r] = *reinterpret_cast<const uint4 *>(p + h0);
                w1[r] = *reinterpret_cast<const uint4 *>(p + h1);
                dw[r] = scale_value(sd[(size_t)srow * ld_d + kb]);
            }
#pragma unroll
            for (int t = 0; t < NT; ++t) {
                if (t < n) {
                    const int8_t *xp = xs.q + (size_t)(xrow0 + t) * k + kb * QK;
                    const uint4 x0 = *reinterpret_cast<const uint4 *>(xp + h0);
                    const uint4 x1 = *reinterpret_cast<const uint4 *>(xp + h1);
                    const float dx = xs.dx[(size_t)(xrow0 + t) * nb + kb];
#pragma unroll
                    for (int r = 0; r < RPW; ++r) {
                        const int s = block_dot(w0[r], w1[r], x0, x1);
                        acc[r][t] = fmaf(dw[r] * dx, small_int_to_float(s), acc[r][t]);
                    }
                }
            }
        }
    }
}

// Sum each of V values (V a power of two, <= 32) over the 32 lanes of a warp
// with a butterfly that halves the values a lane carries at each of the first
// log2(V) levels (V - 1 + 5 - log2(V) shuffles instead of 5 V).  Every value
// is summed over the same xor tree (offsets 16, 8, 4, 2, 1) as warp_sum_all,
// so the results are bitwise those of warp_sum_all.  Lane l returns the sum
// of value reduce_scatter_index<V>(l); the lanes with l % (32 / V) == 0 hold
// the V distinct values.
__host__ __device__ constexpr int pow2_ceil(int v) {
    return v <= 1 ? 1 : v <= 2 ? 2 : v <= 4 ? 4 : v <= 8 ? 8 : v <= 16 ? 16 : 32;
}

template <int V>
__device__ __forceinline__ float warp_reduce_scatter(float (&a)[V]) {
    const int lane = threadIdx.x & 31;
    int m = V;
#pragma unroll
    for (int o = 16; o >= 1; o >>= 1) {
        if (m > 1) {
            const bool upper = (lane & o) != 0;
#pragma unroll
            for (int i = 0; i < V / 2; ++i) {
                if (i < m / 2) {
                    const float send = upper ? a[i] : a[i + m / 2];
                    const float keep = upper ? a[i + m / 2] : a[i];
                    a[i] = keep + __shfl_xor_sync(0xffffffffu, send, o);
                }
            }
            m >>= 1;
        } else {
            a[0] += __shfl_xor_sync(0xffffffffu, a[0], o);
        }
    }
    return a[0];
}

template <int V>
__device__ __forceinline__ int reduce_scatter_index(int lane) {
    int idx = 0, m = V;
#pragma unroll
    for (int o = 16; o >= 1 && m > 1; o >>= 1) {
        if (lane & o) idx += m / 2;
        m >>= 1;
    }
    return idx;
}

// The lowest lane that holds value idx after warp_reduce_scatter<V>: the
// inverse of reduce_scatter_index (bit j of idx, from the top, is lane bit
// 4 - j).
template <int V>
__device__ __forceinline__ int reduce_scatter_lane(int idx) {
    int lane = 0, m = V, o = 16;
#pragma unroll
    for (int j = 0; j < 5 && m > 1; ++j) {
        if (idx & (m / 2)) lane |= o;
        idx &= m / 2 - 1;
        m >>= 1;
        o >>= 1;
    }
    return lane;
}

// Computes this warp's rows of a stage for activation rows [xrow0, xrow0+n)
// and hands each warp sum to emit(row, t, v) (row within the tile, t < NT;
// called by the one lane that holds the sum).
// RPW_ONLY != 0 compiles only that rows-per-warp case (g.rpw must equal it).
// warp_id: the warp's index among the tile's consumer warps (default: its
// index in the CTA).
template <int NT, int RPW_ONLY = 0, class EmitFn>
__device__ __forceinline__ void warp_rows(const int8_t *sq, const uint16_t *sd, int k, int ld_d,
                                          const Geo &g, const XStage &xs, int xrow0, int n,
                                          EmitFn emit, int warp_id = -1) {
    const int warp = warp_id >= 0 ? warp_id : (int)(threadIdx.x >> 5);
    const int lane = threadIdx.x & 31;
    const int seg = warp % g.wpr;
    const int row0 = (warp / g.wpr) * g.rpw;
#define Q8_ROWS_CASE(RPW_)                                                                    \
    {                                                                                         \
        float acc[RPW_][NT];                                                                  \
        dot_rows<NT, RPW_>(sq, sd, k, ld_d, row0, 0, RPW_, seg, g.wpr, xs, xrow0, n, acc);    \
        constexpr int V = RPW_ * NT;                                                          \
        if constexpr (V <= 32) {                                                              \
            constexpr int VP = pow2_ceil(V);                                                  \
            float a[VP];                                                                      \
            _Pragma("unroll") for (int i = 0; i < VP; ++i)                                    \
                a[i] = i < V ? reinterpret_cast<float(&)[V]>(acc)[i] : 0.0f;                  \
            const float v = warp_reduce_scatter<VP>(a);                                       \
            if ((lane & (32 / VP - 1)) == 0) {                                                \
                const int idx = reduce_scatter_index<VP>(lane);                               \
                if (idx < V) {                                                                \
                    const int r = idx / NT, t = idx - (idx / NT) * NT;                        \
                    emit(row0 + r, t, v);                                                     \
                }                                                                             \
            }                                                                                 \
        } else {                                                                              \
            _Pragma("unroll") for (int r = 0; r < RPW_; ++r)                                  \
                _Pragma("unroll") for (int t = 0; t < NT; ++t) {                              \
                    const float v = warp_sum_all(acc[r][t]);                                  \
                    if (lane == 0) emit(row0 + r, t, v);                                      \
                }                                                                             \
        }                                                                                     \
    }
    if constexpr (RPW_ONLY != 0) {
        Q8_ROWS_CASE(RPW_ONLY)
    } else {
        if (g.rpw == 5) Q8_ROWS_CASE(5)
        else if (g.rpw == 4) Q8_ROWS_CASE(4)
        else if (g.rpw == 2) Q8_ROWS_CASE(2)
        else Q8_ROWS_CASE(1)
    }
#undef Q8_ROWS_CASE
}

// Gate/up tile with whole rows per warp (wpr == 1, rpw even): warp w owns
// gate stage rows w*rpw/2 + i and the matching up rows half + w*rpw/2 + i
// (i < rpw/2).  emit(i_row, t, g, u) gets each (gate row within the tile, t)
// with its two final sums, called by one lane.
template <int NT, class EmitFn>
__device__ __forceinline__ void warp_pairs(const int8_t *sq, const uint16_t *sd, int k, int ld_d,
                                           const Geo &g, int half, const XStage &xs, int xrow0,
                                           int n, EmitFn emit, int warp_id = -1) {
    const int warp = warp_id >= 0 ? warp_id : (int)(threadIdx.x >> 5);
    const int lane = threadIdx.x & 31;
#define Q8_PAIRS_CASE(RPW_)                                                                   \
    {                                                                                         \
        constexpr int H = RPW_ / 2;                                                           \
        const int row0 = warp * H;                                                            \
        float acc[RPW_][NT];                                                                  \
        dot_rows<NT, RPW_>(sq, sd, k, ld_d, row0, half + row0, H, 0, 1, xs, xrow0, n, acc);   \
        constexpr int V = RPW_ * NT;                                                          \
        constexpr int VP = pow2_ceil(V);                                                      \
        static_assert(V <= 32, "pair tile too wide");                                         \
        float a[VP];                                                                          \
        _Pragma("unroll") for (int i = 0; i < VP; ++i)                                        \
            a[i] = i < V ? reinterpret_cast<float(&)[V]>(acc)[i] : 0.0f;                      \
        const float v = warp_reduce_scatter<VP>(a);                                           \
        const int idx = reduce_scatter_index<VP>(lane);                                       \
        const int up_idx = idx + H * NT;                                                      \
        const float u = __shfl_sync(0xffffffffu, v,                                           \
                                    reduce_scatter_lane<VP>(up_idx < VP ? up_idx : 0));       \
        if ((lane & (32 / VP - 1)) == 0 && idx < H * NT) {                                    \
            const int i = idx / NT, t = idx - (idx / NT) * NT;                                \
            emit(row0 + i, t, v, u);                                                          \
        }                                                                                     \
    }
    if (g.rpw == 4) Q8_PAIRS_CASE(4)
    else Q8_PAIRS_CASE(2)
#undef Q8_PAIRS_CASE
}

// The warp partial sums of a K-split tile go to part[(row * wpr + seg) * NT + t].
template <int NT>
__device__ __forceinline__ void warp_rows_to_part(const int8_t *sq, const uint16_t *sd, int k,
                                                  int ld_d, const Geo &g, const XStage &xs,
                                                  int xrow0, int n, float *part) {
    const int seg = (threadIdx.x >> 5) % g.wpr;
    warp_rows<NT>(sq, sd, k, ld_d, g, xs, xrow0, n, [&](int row, int t, float v) {
        part[(row * g.wpr + seg) * NT + t] = v;
    });
}

// Calls f(std::integral_constant<int, NTC>) with the smallest NTC in
// {1, 2, 4, 8}, NTC <= NTMAX, that covers n activation rows (n warp-uniform),
// so a pass over few rows pays for few rows.
template <int NTMAX, class F>
__device__ __forceinline__ void with_nt(int n, F &&f) {
    if constexpr (NTMAX >= 8) {
        if (n > 4) {
            f(std::integral_constant<int, 8>{});
            return;
        }
    }
    if constexpr (NTMAX >= 4) {
        if (n > 2) {
            f(std::integral_constant<int, 4>{});
            return;
        }
    }
    if constexpr (NTMAX >= 2) {
        if (n > 1) {
            f(std::integral_constant<int, 2>{});
            return;
        }
    }
    f(std::integral_constant<int, 1>{});
}

// Row sum of tile row `row`, activation t, from the warp partials (seg order).
template <int NT>
__device__ __forceinline__ float part_sum(const float *part, const Geo &g, int row, int t) {
    float v = part[(row * g.wpr) * NT + t];
    for (int sgi = 1; sgi < g.wpr; ++sgi) v += part[(row * g.wpr + sgi) * NT + t];
    return v;
}

// Launch a streaming kernel (kThreadsStream threads) with programmatic stream
// serialization: the kernel itself waits for the preceding grid before it
// reads anything that grid may write.
template <class P>
__host__ inline q8_status launch_stream(void (*kern)(P), int grid, size_t smem, cudaStream_t s,
                                        const P &params, const char *what) {
    // opt in to the full shared memory once per kernel and device (not per
    // launch, so that launches inside a stream capture make no attribute calls)
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64)
        Q8_FAIL(Q8_E_CUDA, "%s: no current device", what);
    if (!smem_opted_in((const void *)kern, dev)) {
        cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             kSmemLimit);
        if (e != cudaSuccess)
            Q8_FAIL(Q8_E_CUDA, "%s: shared-memory attribute: %s", what, cudaGetErrorString(e));
        set_smem_opted_in((const void *)kern, dev);
    }
    if (smem > (size_t)kSmemLimit) Q8_FAIL(Q8_E_UNSUPPORTED, "%s: plan exceeds shared memory", what);
    cudaLaunchConfig_t cfg{};
    cfg.gridDim = dim3((unsigned)grid);
    cfg.blockDim = dim3(kThreadsStream);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    cudaError_t e = cudaLaunchKernelEx(&cfg, kern, params);
    if (e != cudaSuccess) Q8_FAIL(Q8_E_CUDA, "%s: launch: %s", what, cudaGetErrorString(e));
    return Q8_OK;
}

__host__ inline int pick_nt(int64_t rows_per_group) {
    if (rows_per_group <= 1) return 1;
    if (rows_per_group <= 2) return 2;
    if (rows_per_group <= 4) return 4;
    return 8;
}

}  // namespace q8
