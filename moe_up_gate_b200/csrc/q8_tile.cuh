// q8_tile.cuh -- the dp4a row engine shared by the GEMV, mul_mat_id and fused
// up/gate kernels.
//
// A CTA stages up to NT quantized activation rows in shared memory, then its
// warps stream weight rows from HBM: lane l of a warp owns the 32-blocks
// kb = l, l + 32, ... of R rows at once (two 16-byte streaming loads per row
// and block), takes the exact int32 block dot against every staged
// activation row with 8 dp4a, scales it by d_w * d_x (an exact fp32 product of
// two fp16 values) and accumulates in fp32.  A row's sum over blocks is a
// warp shuffle reduction in a fixed order, so results are deterministic.
#pragma once

#include "q8_device.cuh"

namespace q8 {

// Shared-memory staging of NT activation rows: the low and high 16 bytes of
// block kb of row t sit at lo[t * nb + kb] and hi[t * nb + kb] (lanes reading
// consecutive blocks touch consecutive 16-byte words: no bank conflicts);
// dx[t * nb + kb] is the block's fp16 scale as fp32.
struct XStage {
    uint4 *lo;
    uint4 *hi;
    float *dx;
    int nb;
};

__host__ __device__ constexpr int xstage_bytes_per_row(int nb) { return nb * (16 + 16 + 4); }

__device__ __forceinline__ XStage make_xstage(void *smem, int nt, int nb) {
    XStage xs;
    xs.lo = reinterpret_cast<uint4 *>(smem);
    xs.hi = xs.lo + (size_t)nt * nb;
    xs.dx = reinterpret_cast<float *>(xs.hi + (size_t)nt * nb);
    xs.nb = nb;
    return xs;
}

// Copy n Q8_0 rows (row arow[t] of aq/ad) into the stage.  aq rows are k bytes
// apart and 16-byte aligned; ad rows are k/32 scales apart.
__device__ __forceinline__ void stage_q8_rows(const XStage &xs, const int8_t *__restrict__ aq,
                                              const uint16_t *__restrict__ ad, int k,
                                              const int *arow, int n) {
    const int nb = xs.nb;
    for (int i = threadIdx.x; i < n * nb * 2; i += blockDim.x) {
        const int t = i / (2 * nb);
        const int rem = i - t * 2 * nb;
        const int kb = rem >> 1;
        const uint4 v = *reinterpret_cast<const uint4 *>(aq + (int64_t)arow[t] * k + kb * QK +
                                                         (rem & 1) * 16);
        ((rem & 1) ? xs.hi : xs.lo)[t * nb + kb] = v;
    }
    for (int i = threadIdx.x; i < n * nb; i += blockDim.x) {
        const int t = i / nb;
        const int kb = i - t * nb;
        xs.dx[i] = scale_value(ad[(int64_t)arow[t] * nb + kb]);
    }
}

// Quantize n fp32 rows (x rows 0..n-1, k floats apart) straight into the
// stage, one warp per 32-block, by the same rule as the quantize kernel.
__device__ __forceinline__ void stage_f32_rows(const XStage &xs, const float *__restrict__ x, int k,
                                               int n) {
    const int nb = xs.nb;
    const int lane = threadIdx.x & 31;
    const int nwarps = blockDim.x >> 5;
    for (int blk = threadIdx.x >> 5; blk < n * nb; blk += nwarps) {
        const int t = blk / nb;
        const int kb = blk - t * nb;
        const float v = x[(int64_t)t * k + kb * QK + lane];
        const float amax = warp_max_all(fabsf(v));
        const float d32 = block_scale(amax);
        const float id = block_inv_scale(d32);
        const int q = quantize_one(v, id);
        int8_t *dst = reinterpret_cast<int8_t *>(lane < 16 ? xs.lo : xs.hi) + (size_t)blk * 16;
        dst[lane & 15] = (int8_t)q;
        if (lane == 0) xs.dx[blk] = scale_value(scale_bits(d32));
    }
}

// acc[r][t] += sum over this lane's blocks of d_w * d_x * isum, for R weight
// rows (wrow/drow) and the first n (<= NT) staged activation rows.
template <int NT, int R>
__device__ __forceinline__ void dot_rows(const int8_t *const (&wrow)[R],
                                         const uint16_t *const (&drow)[R], const XStage &xs,
                                         int n, int lane, float (&acc)[R][NT]) {
    const int nb = xs.nb;
#pragma unroll 2
    for (int kb = lane; kb < nb; kb += 32) {
        uint4 w0[R], w1[R];
        float dw[R];
#pragma unroll
        for (int r = 0; r < R; ++r) {
            const int8_t *p = wrow[r] + kb * QK;
            w0[r] = ld_stream_v4(p);
            w1[r] = ld_stream_v4(p + 16);
            dw[r] = scale_value(ld_stream_u16(drow[r] + kb));
        }
#pragma unroll
        for (int t = 0; t < NT; ++t) {
            if (t < n) {
                const uint4 x0 = xs.lo[t * nb + kb];
                const uint4 x1 = xs.hi[t * nb + kb];
                const float dx = xs.dx[t * nb + kb];
#pragma unroll
                for (int r = 0; r < R; ++r) {
                    const int s = block_dot(w0[r], w1[r], x0, x1);
                    acc[r][t] = fmaf(dw[r] * dx, (float)s, acc[r][t]);
                }
            }
        }
    }
}

template <int NT, int R>
__device__ __forceinline__ void reduce_rows(float (&acc)[R][NT]) {
#pragma unroll
    for (int r = 0; r < R; ++r)
#pragma unroll
        for (int t = 0; t < NT; ++t) acc[r][t] = warp_sum_all(acc[r][t]);
}

// Rows [row0, row_end) of one matrix (wq/wd at the matrix's first row) times
// the n staged rows; y[pair[t] * rows + r] = result.  Each warp takes groups
// of R consecutive rows.
template <int NT, int R>
__device__ __forceinline__ void run_rows(const int8_t *__restrict__ wq,
                                         const uint16_t *__restrict__ wd, int k, int64_t ld_d,
                                         int rows, int row0, int row_end, const XStage &xs, int n,
                                         const int *pair, float *__restrict__ y) {
    const int lane = threadIdx.x & 31;
    const int warp = threadIdx.x >> 5;
    const int nwarps = blockDim.x >> 5;
    for (int rg = row0 + warp * R; rg < row_end; rg += nwarps * R) {
        const int8_t *wrow[R];
        const uint16_t *drow[R];
#pragma unroll
        for (int r = 0; r < R; ++r) {
            const int rr = min(rg + r, row_end - 1);
            wrow[r] = wq + (int64_t)rr * k;
            drow[r] = wd + (int64_t)rr * ld_d;
        }
        float acc[R][NT];
#pragma unroll
        for (int r = 0; r < R; ++r)
#pragma unroll
            for (int t = 0; t < NT; ++t) acc[r][t] = 0.0f;
        dot_rows<NT, R>(wrow, drow, xs, n, lane, acc);
        reduce_rows<NT, R>(acc);
#pragma unroll
        for (int r = 0; r < R; ++r)
#pragma unroll
            for (int t = 0; t < NT; ++t)
                if (lane == ((r * NT + t) & 31) && t < n && rg + r < row_end)
                    y[(int64_t)pair[t] * rows + rg + r] = acc[r][t];
    }
}

}  // namespace q8
