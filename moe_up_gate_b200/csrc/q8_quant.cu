// q8_quant.cu -- Q8_0 quantization kernels (q8_quantize_row, q8_pack) and the
// library's common host helpers (status strings, error detail, validation).
//
// The quantizer is the activation quantizer of the news.hada.io article on
// Gemma 4 26B-A4B Q8_0 (section 「3段階で構成された修正」, quantize_row_q8_0_x4),
// in its plain one-row form; weights are packed with the same rule.
#include <stdarg.h>
#include <stdio.h>

#include <mutex>
#include <set>
#include <utility>

#include "q8_device.cuh"
#include "q8_internal.h"
#include "q8_ptx.cuh"

namespace q8 {

static thread_local char g_detail[512] = "";

void set_error_detail(const char *fmt, ...) {
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(g_detail, sizeof g_detail, fmt, ap);
    va_end(ap);
}

static std::mutex g_optin_mu;
static std::set<std::pair<const void *, int>> g_optin;

bool smem_opted_in(const void *kernel, int device) {
    std::lock_guard<std::mutex> lock(g_optin_mu);
    return g_optin.count({kernel, device}) != 0;
}

void set_smem_opted_in(const void *kernel, int device) {
    std::lock_guard<std::mutex> lock(g_optin_mu);
    g_optin.insert({kernel, device});
}

q8_status check_tensor(const q8_tensor *W, const char *name, bool need_single) {
    Q8_REQUIRE(W != nullptr, Q8_E_NULL, "%s: tensor view is NULL", name);
    Q8_REQUIRE(W->qs != nullptr && W->d != nullptr, Q8_E_NULL, "%s: qs or d is NULL", name);
    Q8_REQUIRE(W->k > 0 && W->k % QK == 0 && W->k <= Q8_MAX_K, Q8_E_SHAPE,
               "%s: k=%lld must be a positive multiple of 32 and <= %d", name, (long long)W->k,
               Q8_MAX_K);
    Q8_REQUIRE(W->rows > 0 && W->rows <= (int64_t)1 << 30, Q8_E_SHAPE, "%s: rows=%lld out of range",
               name, (long long)W->rows);
    Q8_REQUIRE(W->n_mat > 0 && W->n_mat <= 65535, Q8_E_SHAPE, "%s: n_mat=%lld out of range", name,
               (long long)W->n_mat);
    Q8_REQUIRE(!need_single || W->n_mat == 1, Q8_E_SHAPE, "%s: n_mat must be 1 here", name);
    Q8_REQUIRE(W->ld_d >= W->k / QK && W->ld_d % 8 == 0, Q8_E_ALIGN,
               "%s: ld_d=%lld must be >= k/32 and a multiple of 8", name, (long long)W->ld_d);
    Q8_REQUIRE(W->mat_stride >= W->rows, Q8_E_SHAPE, "%s: mat_stride < rows", name);
    Q8_REQUIRE(aligned16(W->qs) && aligned16(W->d), Q8_E_ALIGN,
               "%s: qs and d must be 16-byte aligned", name);
    return Q8_OK;
}

// ---------------------------------------------------------------------------
// Quantize rows of length k.  Eight threads own one 32-block (four floats
// each, one 16-byte load); the block amax is a 3-step shuffle max.  Output
// quants are dense [n_rows][k]; scales go to d[row * ld_d + b].
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(256) quantize_rows_kernel(const float *__restrict__ x,
                                                            int64_t n_rows, int k,
                                                            int8_t *__restrict__ qs,
                                                            uint16_t *__restrict__ d,
                                                            int64_t ld_d, int early) {
    // x may come from the previous kernel, which may also still read qs/d
    griddep_wait();
    // Activation rows (early != 0) let the next kernel launch at once.  Packed
    // weights do not: a streaming kernel prefetches weights before it waits.
    if (early) griddep_launch_dependents();
    const int lane = threadIdx.x & 31;
    const int64_t nb = k / QK;
    const int64_t total8 = n_rows * nb * 8;
    const int64_t stride = (int64_t)gridDim.x * blockDim.x;
    for (int64_t base = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) & ~31LL; base < total8;
         base += stride) {
        const int64_t g = base + lane;
        const bool ok = g < total8;
        const int64_t blk = g >> 3;
        const int part = (int)(g & 7);
        const int64_t row = ok ? blk / nb : 0;
        const int64_t b = ok ? blk - row * nb : 0;
        const int64_t off = row * k + b * QK + part * 4;
        float4 v = ok ? *reinterpret_cast<const float4 *>(x + off) : make_float4(0.f, 0.f, 0.f, 0.f);
        float a = fmaxf(fmaxf(fabsf(v.x), fabsf(v.y)), fmaxf(fabsf(v.z), fabsf(v.w)));
        a = fmaxf(a, __shfl_xor_sync(0xffffffffu, a, 1));
        a = fmaxf(a, __shfl_xor_sync(0xffffffffu, a, 2));
        a = fmaxf(a, __shfl_xor_sync(0xffffffffu, a, 4));
        const float d32 = block_scale(a);
        const float id = block_inv_scale(d32);
        char4 q;
        q.x = (signed char)quantize_one(v.x, id);
        q.y = (signed char)quantize_one(v.y, id);
        q.z = (signed char)quantize_one(v.z, id);
        q.w = (signed char)quantize_one(v.w, id);
        if (ok) {
            *reinterpret_cast<char4 *>(qs + off) = q;
            if (part == 0) d[row * ld_d + b] = scale_bits(d32);
        }
    }
}

q8_status launch_quantize(const float *x, int64_t n_rows, int64_t k, int8_t *qs,
                                 uint16_t *d, int64_t ld_d, cudaStream_t s, bool weights) {
    const int64_t total8 = n_rows * (k / QK) * 8;
    int64_t blocks = (total8 + 255) / 256;
    if (blocks > 148 * 16) blocks = 148 * 16;
    if (blocks < 1) blocks = 1;
    return launch_pdl("quantize_rows_kernel", quantize_rows_kernel, dim3((unsigned)blocks),
                      dim3(256), 0, s, x, n_rows, (int)k, qs, d, ld_d, weights ? 0 : 1);
}

}  // namespace q8

using namespace q8;

extern "C" {

int64_t q8_scale_stride(int64_t k) {
    if (k <= 0 || k % QK) return 0;
    return (k / QK + 7) / 8 * 8;
}

q8_status q8_quantize_row(const float *x, int64_t n_rows, int64_t k, int8_t *qs, uint16_t *d,
                          void *stream) {
    Q8_REQUIRE(x && qs && d, Q8_E_NULL, "q8_quantize_row: NULL pointer");
    Q8_REQUIRE(n_rows >= 1 && n_rows <= ((int64_t)1 << 31), Q8_E_SHAPE,
               "q8_quantize_row: n_rows=%lld", (long long)n_rows);
    Q8_REQUIRE(k > 0 && k % QK == 0 && k <= Q8_MAX_K, Q8_E_SHAPE,
               "q8_quantize_row: k=%lld must be a positive multiple of 32 <= %d", (long long)k,
               Q8_MAX_K);
    Q8_REQUIRE(aligned16(x), Q8_E_ALIGN, "q8_quantize_row: x must be 16-byte aligned");
    Q8_REQUIRE(((uintptr_t)qs & 3u) == 0, Q8_E_ALIGN, "q8_quantize_row: qs must be 4-byte aligned");
    Q8_REQUIRE(((uintptr_t)d & 1u) == 0, Q8_E_ALIGN, "q8_quantize_row: d must be 2-byte aligned");
    return launch_quantize(x, n_rows, k, qs, d, k / QK, (cudaStream_t)stream, false);
}

q8_status q8_pack(const float *w, int64_t n_rows, int64_t k, int8_t *qs, uint16_t *d,
                  int64_t ld_d, void *stream) {
    Q8_REQUIRE(w && qs && d, Q8_E_NULL, "q8_pack: NULL pointer");
    Q8_REQUIRE(n_rows >= 1 && n_rows <= ((int64_t)1 << 34), Q8_E_SHAPE, "q8_pack: n_rows=%lld",
               (long long)n_rows);
    Q8_REQUIRE(k > 0 && k % QK == 0 && k <= Q8_MAX_K, Q8_E_SHAPE,
               "q8_pack: k=%lld must be a positive multiple of 32 <= %d", (long long)k, Q8_MAX_K);
    Q8_REQUIRE(ld_d >= k / QK && ld_d % 8 == 0, Q8_E_ALIGN,
               "q8_pack: ld_d=%lld must be >= k/32 and a multiple of 8", (long long)ld_d);
    Q8_REQUIRE(aligned16(w) && aligned16(qs) && aligned16(d), Q8_E_ALIGN,
               "q8_pack: w, qs and d must be 16-byte aligned");
    cudaStream_t s = (cudaStream_t)stream;
    if (ld_d > k / QK) {
        cudaError_t e = cudaMemsetAsync(d, 0, (size_t)n_rows * ld_d * sizeof(uint16_t), s);
        if (e != cudaSuccess) Q8_FAIL(Q8_E_CUDA, "q8_pack: memset: %s", cudaGetErrorString(e));
    }
    return launch_quantize(w, n_rows, k, qs, d, ld_d, s, true);
}

q8_status q8_pack_up_gate(const float *w_gate, const float *w_up, int64_t n_mat, int64_t n_ff,
                          int64_t k, int8_t *qs, uint16_t *d, int64_t ld_d, void *stream) {
    Q8_REQUIRE(w_gate && w_up && qs && d, Q8_E_NULL, "q8_pack_up_gate: NULL pointer");
    Q8_REQUIRE(n_mat >= 1 && n_mat <= 65535, Q8_E_SHAPE, "q8_pack_up_gate: n_mat=%lld",
               (long long)n_mat);
    Q8_REQUIRE(n_ff >= QK && n_ff % QK == 0 && n_ff <= ((int64_t)1 << 29), Q8_E_SHAPE,
               "q8_pack_up_gate: n_ff=%lld must be a positive multiple of 32", (long long)n_ff);
    Q8_REQUIRE(k > 0 && k % QK == 0 && k <= Q8_MAX_K, Q8_E_SHAPE,
               "q8_pack_up_gate: k=%lld must be a positive multiple of 32 <= %d", (long long)k,
               Q8_MAX_K);
    Q8_REQUIRE(ld_d >= k / QK && ld_d % 8 == 0, Q8_E_ALIGN,
               "q8_pack_up_gate: ld_d=%lld must be >= k/32 and a multiple of 8", (long long)ld_d);
    Q8_REQUIRE(aligned16(w_gate) && aligned16(w_up) && aligned16(qs) && aligned16(d), Q8_E_ALIGN,
               "q8_pack_up_gate: w_gate, w_up, qs and d must be 16-byte aligned");
    cudaStream_t s = (cudaStream_t)stream;
    if (ld_d > k / QK) {
        cudaError_t e =
            cudaMemsetAsync(d, 0, (size_t)n_mat * 2 * n_ff * ld_d * sizeof(uint16_t), s);
        if (e != cudaSuccess) Q8_FAIL(Q8_E_CUDA, "q8_pack_up_gate: memset: %s", cudaGetErrorString(e));
    }
    // each matrix: its gate rows to rows 0..n_ff-1, its up rows to n_ff..2*n_ff-1
    // (offsets are multiples of k floats / k bytes / ld_d scales: 16-byte aligned)
    for (int64_t m = 0; m < n_mat; ++m) {
        const int64_t r0 = m * 2 * n_ff;
        q8_status st = launch_quantize(w_gate + m * n_ff * k, n_ff, k, qs + r0 * k, d + r0 * ld_d,
                                       ld_d, s, true);
        if (st != Q8_OK) return st;
        st = launch_quantize(w_up + m * n_ff * k, n_ff, k, qs + (r0 + n_ff) * k,
                             d + (r0 + n_ff) * ld_d, ld_d, s, true);
        if (st != Q8_OK) return st;
    }
    return Q8_OK;
}

const char *q8_status_string(q8_status st) {
    switch (st) {
        case Q8_OK: return "ok";
        case Q8_E_NULL: return "null pointer";
        case Q8_E_SHAPE: return "bad shape";
        case Q8_E_ALIGN: return "misaligned pointer or stride";
        case Q8_E_BAD_ID: return "routing id out of range or repeated";
        case Q8_E_UNSUPPORTED: return "unsupported request";
        case Q8_E_CUDA: return "CUDA error";
        case Q8_E_WORKSPACE: return "workspace missing or too small";
    }
    return "unknown status";
}

const char *q8_last_error(void) { return g_detail; }

}  // extern "C"
