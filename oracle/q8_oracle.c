/*
 * q8_oracle.c -- plain scalar CPU oracle for the Q8_0 decode path and the
 * fused MoE up/gate + SwiGLU step.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing in the product path (the CUDA library
 * under moe_up_gate_b200/) may include, link or call this file.  Only the
 * tests, __graft_entry__.smoke() and bench.py's CPU-baseline leg use it.  It
 * shares no code, header, table or constant with the CUDA path.
 *
 * Every function is the plain definition written out, one scalar loop at a
 * time, with no blocking, fusion or reordering beyond what the definition
 * states.  Floating-point sums are carried in fp64; the per-block integer
 * dot products are exact int32.
 *
 * Sources (the web pages this method is taken from):
 *  - "GPUなしで13年前のXeon上でGemma 4 26Bを毎秒5トークンで実行する"
 *    (news.hada.io), sections 「非AVX2ビルドで壊れていた演算パス」 and
 *    「3段階で構成された修正」: the MOE_FUSED_UP_GATE / FUSED_UP_GATE ops,
 *    the combined up_gate_exps weight [n_embd, 2*n_ff, n_experts] whose first
 *    half is gate and second half is up, the two view_3d slices, the per-slice
 *    mul_mat_id and fused_mul_unary(gate, up, SILU); the Q8_0 x Q8_0 block dot
 *    (ggml_vec_dot_q8_0_q8_0) and the Q8_0 activation quantizer
 *    (quantize_row_q8_0_x4).
 *  - "narray-llm" README, section "Llama 2 110M を int8 (Q8_0) で": Q8_0
 *    single-token decode.
 *  The pages name Q8_0 but never print its layout.  The reading used here:
 *  blocks of 32 int8 values along the contiguous axis, one fp16 scale per
 *  block, d = amax/127 computed in fp32 and stored as fp16 (round to nearest
 *  even, subnormals kept), q = round-half-away-from-zero(x * (1/d)).
 *
 * Parity pins for every function here live in tests/test_oracle_*.py.  No
 * function is "parity unpinned".
 *
 * Build: gcc -O2 -std=c11 -fPIC -shared -fopenmp -ffp-contract=off
 *        (no -ffast-math: the fp32 steps of the quantizer must be IEEE).
 */
#include <math.h>
#include <stdint.h>
#include <stddef.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

#define QK 32 /* weights per Q8_0 block */

/* ------------------------------------------------------------------------ */
/* IEEE-754 binary16 <-> binary32, written from the format definition.      */
/* ------------------------------------------------------------------------ */

/* fp32 -> fp16 bits, round to nearest, ties to even; fp16 subnormals kept;
 * overflow to infinity; NaN stays NaN (quiet). */
uint16_t oracle_fp16_from_fp32(float f)
{
    uint32_t x;
    memcpy(&x, &f, sizeof x);
    uint32_t sign = (x >> 16) & 0x8000u;
    uint32_t bexp = (x >> 23) & 0xffu;
    uint32_t man = x & 0x7fffffu;

    if (bexp == 0xffu) /* inf or NaN */
        return (uint16_t)(sign | 0x7c00u | (man ? 0x0200u : 0u));
    if (bexp == 0u) /* fp32 zero or subnormal: far below half of 2^-24 */
        return (uint16_t)sign;

    int e = (int)bexp - 127; /* value = 1.man * 2^e */
    if (e > 15)
        return (uint16_t)(sign | 0x7c00u);

    if (e >= -14) { /* lands in the fp16 normal range: drop 13 mantissa bits */
        uint32_t keep = man >> 13;
        uint32_t rest = man & 0x1fffu;
        uint32_t h = ((uint32_t)(e + 15) << 10) | keep;
        if (rest > 0x1000u || (rest == 0x1000u && (keep & 1u)))
            h += 1u; /* a carry may step the exponent, or reach infinity */
        return (uint16_t)(sign | h);
    }

    /* fp16 subnormal: value / 2^-24 = (2^23 + man) * 2^(e+1) */
    if (e < -25)
        return (uint16_t)sign; /* below 2^-25: nearer to zero than to 2^-24 */
    uint32_t sig = 0x800000u | man;
    int shift = -(e + 1); /* 14 .. 24 */
    uint32_t q = sig >> shift;
    uint32_t rem = sig & ((1u << shift) - 1u);
    uint32_t half = 1u << (shift - 1);
    if (rem > half || (rem == half && (q & 1u)))
        q += 1u; /* may become 0x400, the smallest normal: same encoding */
    return (uint16_t)(sign | q);
}

/* fp16 bits -> fp32 value (exact: every binary16 value is a binary32 value). */
float oracle_fp32_from_fp16(uint16_t h)
{
    int e = (h >> 10) & 0x1f;
    int m = h & 0x3ff;
    double v;
    if (e == 0)
        v = ldexp((double)m, -24);
    else if (e == 31)
        v = m ? (double)NAN : (double)INFINITY;
    else
        v = ldexp((double)(1024 + m), e - 25);
    return (float)((h & 0x8000u) ? -v : v);
}

/* Element-wise array forms of the two conversions above. */
void oracle_fp16_from_fp32_n(const float *f, int64_t n, uint16_t *h)
{
    for (int64_t i = 0; i < n; ++i)
        h[i] = oracle_fp16_from_fp32(f[i]);
}

void oracle_fp32_from_fp16_n(const uint16_t *h, int64_t n, float *f)
{
    for (int64_t i = 0; i < n; ++i)
        f[i] = oracle_fp32_from_fp16(h[i]);
}

/* ------------------------------------------------------------------------ */
/* Q8_0 quantization of one row (quantize_row_q8_0, plain row version).     */
/* ------------------------------------------------------------------------ */

/* x[k] fp32 -> q[k] int8, d[k/32] fp16 bits.  k must be a multiple of 32.
 * Per block: amax = max |x_i|; d32 = amax / 127 (fp32 IEEE division);
 * id = 1/d32 (0 when d32 == 0); q_i = round-half-away(x_i * id); d = fp16(d32).
 * Returns 0, or -1 if some |q_i| > 127 (cannot happen for finite x). */
int oracle_quantize_row(const float *x, int64_t k, int8_t *q, uint16_t *d)
{
    int bad = 0;
    for (int64_t b = 0; b < k / QK; ++b) {
        const float *xb = x + b * QK;
        float amax = 0.0f;
        for (int i = 0; i < QK; ++i) {
            float a = fabsf(xb[i]);
            if (a > amax)
                amax = a;
        }
        float d32 = amax / 127.0f;
        float id = (d32 != 0.0f) ? 1.0f / d32 : 0.0f;
        for (int i = 0; i < QK; ++i) {
            float v = xb[i] * id;
            float r = roundf(v); /* C roundf: halfway cases away from zero */
            if (r > 127.0f || r < -127.0f)
                bad = 1;
            q[b * QK + i] = (int8_t)r;
        }
        d[b] = oracle_fp16_from_fp32(d32);
    }
    return bad ? -1 : 0;
}

/* Quantize n_rows rows of length k (row stride k floats). */
int oracle_quantize_rows(const float *x, int64_t n_rows, int64_t k, int8_t *q, uint16_t *d)
{
    int bad = 0;
    for (int64_t r = 0; r < n_rows; ++r)
        if (oracle_quantize_row(x + r * k, k, q + r * k, d + r * (k / QK)))
            bad = 1;
    return bad ? -1 : 0;
}

/* ------------------------------------------------------------------------ */
/* Block dot (ggml_vec_dot_q8_0_q8_0) and the row result.                   */
/* ------------------------------------------------------------------------ */

/* isum = sum_{i<32} a_i * b_i, exact in int32 (|isum| <= 32*127*127). */
int32_t oracle_block_dot(const int8_t *a, const int8_t *b)
{
    int32_t s = 0;
    for (int i = 0; i < QK; ++i)
        s += (int32_t)a[i] * (int32_t)b[i];
    return s;
}

/* y = sum_b fp32(dw_b) * fp32(dx_b) * isum_b, accumulated in fp64 over the
 * k/32 blocks of one weight row and one activation row. */
double oracle_row_dot(const int8_t *qw, const uint16_t *dw, const int8_t *qx,
                      const uint16_t *dx, int64_t k)
{
    double s = 0.0;
    for (int64_t b = 0; b < k / QK; ++b) {
        int32_t isum = oracle_block_dot(qw + b * QK, qx + b * QK);
        s += (double)oracle_fp32_from_fp16(dw[b]) * (double)oracle_fp32_from_fp16(dx[b]) *
             (double)isum;
    }
    return s;
}

/* Per-block int32 dots of weight row r with activation row x, all blocks. */
void oracle_row_block_dots(const int8_t *qw, const int8_t *qx, int64_t k, int32_t *isum)
{
    for (int64_t b = 0; b < k / QK; ++b)
        isum[b] = oracle_block_dot(qw + b * QK, qx + b * QK);
}

/* ------------------------------------------------------------------------ */
/* GEMV: y[t][r] = W[r] . x[t]  (W: qs [rows][k], d [rows][k/32]).          */
/* ------------------------------------------------------------------------ */
void oracle_gemv(const int8_t *wq, const uint16_t *wd, int64_t rows, int64_t k,
                 const int8_t *xq, const uint16_t *xd, int64_t n_tok, double *y)
{
    const int64_t nb = k / QK;
#pragma omp parallel for schedule(static)
    for (int64_t r = 0; r < rows; ++r)
        for (int64_t t = 0; t < n_tok; ++t)
            y[t * rows + r] = oracle_row_dot(wq + r * k, wd + r * nb, xq + t * k, xd + t * nb, k);
}

/* ------------------------------------------------------------------------ */
/* Fused MoE up/gate + SwiGLU (MOE_FUSED_UP_GATE; FUSED_UP_GATE when dense). */
/* ------------------------------------------------------------------------ */

/* silu(z) = z * sigmoid(z) = z / (1 + exp(-z)), in fp64. */
double oracle_silu(double z) { return z / (1.0 + exp(-z)); }

/* up_gate: qs [n_exp][2*n_ff][n_embd], d [n_exp][2*n_ff][n_embd/32].
 * Rows 0..n_ff-1 of each expert are gate, rows n_ff..2*n_ff-1 are up.
 * x: [n_tok][n_embd] quantized.  ids: [n_tok][n_used] expert ids, or NULL for
 * the dense op (n_exp == 1, n_used == 1, every token uses matrix 0).
 * For each (t, k): e = ids[t][k]; for r < n_ff:
 *   g = W_e[r] . x_t ; u = W_e[n_ff + r] . x_t ; h = silu(g) * u.
 * g, u, h: [n_tok][n_used][n_ff] fp64 (g, u may be NULL).
 * Returns 0, or -1 on an id outside [0, n_exp) (that pair is left unwritten). */
int oracle_up_gate_swiglu(const int8_t *wq, const uint16_t *wd, int64_t n_exp, int64_t n_ff,
                          int64_t n_embd, const int8_t *xq, const uint16_t *xd, int64_t n_tok,
                          const int32_t *ids, int64_t n_used, double *g, double *u, double *h)
{
    const int64_t nb = n_embd / QK;
    int bad = 0;
    for (int64_t t = 0; t < n_tok; ++t) {
        for (int64_t s = 0; s < n_used; ++s) {
            int64_t e = ids ? (int64_t)ids[t * n_used + s] : 0;
            if (e < 0 || e >= n_exp) {
                bad = 1;
                continue;
            }
            const int8_t *we = wq + e * (2 * n_ff) * n_embd;
            const uint16_t *de = wd + e * (2 * n_ff) * nb;
            const int64_t o = (t * n_used + s) * n_ff;
#pragma omp parallel for schedule(static)
            for (int64_t r = 0; r < n_ff; ++r) {
                double gv = oracle_row_dot(we + r * n_embd, de + r * nb, xq + t * n_embd,
                                           xd + t * nb, n_embd);
                double uv = oracle_row_dot(we + (n_ff + r) * n_embd, de + (n_ff + r) * nb,
                                           xq + t * n_embd, xd + t * nb, n_embd);
                if (g)
                    g[o + r] = gv;
                if (u)
                    u[o + r] = uv;
                h[o + r] = oracle_silu(gv) * uv;
            }
        }
    }
    return bad ? -1 : 0;
}

/* The fused multiply-unary of the path with separate gate and up weights
 * (page "GPUなしで13年前のXeon上でGemma 4 26Bを毎秒5トークンで実行する",
 * section 「3段階で構成された修正」, runtime graph fallback): when the gate
 * and up weights are already separate tensors, two mul_mat_id products g and
 * u are joined by one SILU-and-multiply op.  h[i] = silu(g[i]) * u[i], fp64. */
void oracle_swiglu(const double *g, const double *u, int64_t n, double *h)
{
    for (int64_t i = 0; i < n; ++i)
        h[i] = oracle_silu(g[i]) * u[i];
}

/* ------------------------------------------------------------------------ */
/* mul_mat_id: y[t][k] = W[ids[t][k]] . a(t, k)                              */
/* ------------------------------------------------------------------------ */

/* W: qs [n_mat][rows][k], d [n_mat][rows][k/32].
 * a: [n_tok][n_used][k] when a_per_slot, else [n_tok][k] (every slot of a
 * token reads the token's row).  ids: [n_tok][n_used].
 * y: [n_tok][n_used][rows] fp64.  Returns -1 on an out-of-range id. */
int oracle_mul_mat_id(const int8_t *wq, const uint16_t *wd, int64_t n_mat, int64_t rows,
                      int64_t k, const int8_t *aq, const uint16_t *ad, int a_per_slot,
                      int64_t n_tok, const int32_t *ids, int64_t n_used, double *y)
{
    const int64_t nb = k / QK;
    int bad = 0;
    for (int64_t t = 0; t < n_tok; ++t) {
        for (int64_t s = 0; s < n_used; ++s) {
            int64_t e = (int64_t)ids[t * n_used + s];
            if (e < 0 || e >= n_mat) {
                bad = 1;
                continue;
            }
            int64_t arow = a_per_slot ? (t * n_used + s) : t;
            const int8_t *we = wq + e * rows * k;
            const uint16_t *de = wd + e * rows * nb;
            double *yo = y + (t * n_used + s) * rows;
#pragma omp parallel for schedule(static)
            for (int64_t r = 0; r < rows; ++r)
                yo[r] = oracle_row_dot(we + r * k, de + r * nb, aq + arow * k, ad + arow * nb, k);
        }
    }
    return bad ? -1 : 0;
}

/* ------------------------------------------------------------------------ */
/* Combine: out[t] = sum_k p[t][k] * y[t][k], k ascending, fp64.             */
/* ------------------------------------------------------------------------ */
void oracle_combine(const double *y, const float *p, int64_t n_tok, int64_t n_used,
                    int64_t n_out, double *out)
{
    for (int64_t t = 0; t < n_tok; ++t)
        for (int64_t r = 0; r < n_out; ++r) {
            double s = 0.0;
            for (int64_t k = 0; k < n_used; ++k)
                s += (double)p[t * n_used + k] * y[(t * n_used + k) * n_out + r];
            out[t * n_out + r] = s;
        }
}

/* ------------------------------------------------------------------------ */
/* Brute force: dequantize both operands to fp64 and multiply plainly.       */
/* ------------------------------------------------------------------------ */
void oracle_dequant_fp64_matmul(const int8_t *wq, const uint16_t *wd, int64_t rows, int64_t k,
                                const int8_t *xq, const uint16_t *xd, int64_t n_tok, double *y)
{
    const int64_t nb = k / QK;
    for (int64_t t = 0; t < n_tok; ++t)
        for (int64_t r = 0; r < rows; ++r) {
            double s = 0.0;
            for (int64_t i = 0; i < k; ++i) {
                double w = (double)oracle_fp32_from_fp16(wd[r * nb + i / QK]) * (double)wq[r * k + i];
                double x = (double)oracle_fp32_from_fp16(xd[t * nb + i / QK]) * (double)xq[t * k + i];
                s += w * x;
            }
            y[t * rows + r] = s;
        }
}

/* ------------------------------------------------------------------------ */
/* The whole MoE feed-forward step, from fp32 x.                              */
/* ------------------------------------------------------------------------ */

/* x [n_tok][n_embd] fp32 -> quantize -> up_gate + SwiGLU -> h rounded to fp32
 * -> quantize per (t, slot) row -> down mul_mat_id -> combine with p (or, when
 * p is NULL, out = the slot-0 result, the dense case with n_used == 1).
 * Scratch buffers are the caller's:
 *   xq [n_tok*n_embd], xd [n_tok*n_embd/32], h [n_tok*n_used*n_ff] (double),
 *   hf [same] (float), hq [same] int8, hd [n_tok*n_used*n_ff/32],
 *   y [n_tok*n_used*n_embd] (double).  out: [n_tok][n_embd] fp64. */
int oracle_moe_ffn(const int8_t *ugq, const uint16_t *ugd, const int8_t *dnq, const uint16_t *dnd,
                   int64_t n_exp, int64_t n_embd, int64_t n_ff, const float *x, int64_t n_tok,
                   const int32_t *ids, const float *p, int64_t n_used, int8_t *xq, uint16_t *xd,
                   double *h, float *hf, int8_t *hq, uint16_t *hd, double *y, double *out)
{
    int rc = 0;
    rc |= oracle_quantize_rows(x, n_tok, n_embd, xq, xd);
    rc |= oracle_up_gate_swiglu(ugq, ugd, n_exp, n_ff, n_embd, xq, xd, n_tok, ids, n_used, NULL,
                                NULL, h);
    for (int64_t i = 0; i < n_tok * n_used * n_ff; ++i)
        hf[i] = (float)h[i];
    rc |= oracle_quantize_rows(hf, n_tok * n_used, n_ff, hq, hd);
    if (ids) {
        rc |= oracle_mul_mat_id(dnq, dnd, n_exp, n_embd, n_ff, hq, hd, 1, n_tok, ids, n_used, y);
    } else {
        oracle_gemv(dnq, dnd, n_embd, n_ff, hq, hd, n_tok, y);
    }
    if (p) {
        oracle_combine(y, p, n_tok, n_used, n_embd, out);
    } else {
        for (int64_t i = 0; i < n_tok * n_embd; ++i)
            out[i] = y[i];
    }
    return rc ? -1 : 0;
}

/* Threads used by the OpenMP loops above (results do not depend on it). */
void oracle_set_num_threads(int n)
{
#ifdef _OPENMP
    if (n > 0)
        omp_set_num_threads(n);
#else
    (void)n;
#endif
}

int oracle_get_max_threads(void)
{
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}
