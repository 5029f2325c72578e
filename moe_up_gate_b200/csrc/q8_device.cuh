// q8_device.cuh -- device building blocks shared by the libq8 kernels:
// the Q8_0 block quantizer, the exact int32 block dot, streaming loads and
// warp reductions.  sm_100a only.
//
// The Q8_0 rule (the pages name the format and its quantizer but print no
// layout; this is the reading the whole library follows): per block of 32,
// amax = max|x|, d32 = amax / 127 in fp32, id = 1 / d32 (0 when d32 == 0),
// q = round-half-away-from-zero(x * id), stored scale = fp16 RNE of d32.
// The dot of a weight block and an activation block is the exact int32
// sum of q_w * q_x; a row result is sum_b d_w,b * d_x,b * isum_b.
#pragma once

#include <cuda_fp16.h>
#include <stdint.h>

namespace q8 {

constexpr int QK = 32;

// ---------------------------------------------------------------------------
// quantization of one 32-block
// ---------------------------------------------------------------------------

// d32 = amax / 127 with IEEE division; id = 1 / d32 with IEEE reciprocal.
__device__ __forceinline__ float block_scale(float amax) { return __fdiv_rn(amax, 127.0f); }
__device__ __forceinline__ float block_inv_scale(float d32) {
    return d32 != 0.0f ? __frcp_rn(d32) : 0.0f;
}
// q = round-half-away-from-zero(x * id); |q| <= 127 for finite x.
__device__ __forceinline__ int quantize_one(float x, float id) {
    return (int)roundf(__fmul_rn(x, id));
}
__device__ __forceinline__ uint16_t scale_bits(float d32) {
    return __half_as_ushort(__float2half_rn(d32));
}
__device__ __forceinline__ float scale_value(uint16_t bits) {
    return __half2float(__ushort_as_half(bits));
}

// One 32-block held by one thread (v[0..31]) quantized by the rule above:
// the codes packed four per word (byte i of word w is element 4w + i);
// returns d32.  amax is the exact maximum of |v|, as in the warp form.
__device__ __forceinline__ float quantize_block_thread(const float (&v)[32], uint32_t (&q)[8]) {
    float amax = 0.0f;
#pragma unroll
    for (int i = 0; i < 32; ++i) amax = fmaxf(amax, fabsf(v[i]));
    const float d32 = block_scale(amax);
    const float id = block_inv_scale(d32);
#pragma unroll
    for (int w = 0; w < 8; ++w) {
        uint32_t word = 0;
#pragma unroll
        for (int b = 0; b < 4; ++b)
            word |= ((uint32_t)quantize_one(v[4 * w + b], id) & 0xffu) << (8 * b);
        q[w] = word;
    }
    return d32;
}

// ---------------------------------------------------------------------------
// warp helpers
// ---------------------------------------------------------------------------
__device__ __forceinline__ float warp_max_all(float v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
    return v;
}

__device__ __forceinline__ float warp_sum_all(float v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}

// ---------------------------------------------------------------------------
// loads
// ---------------------------------------------------------------------------

// Weights are read once per call: streaming (evict-first) 16-byte loads.
__device__ __forceinline__ uint4 ld_stream_v4(const void *p) {
    uint4 r;
    asm volatile("ld.global.cs.v4.u32 {%0, %1, %2, %3}, [%4];"
                 : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
                 : "l"(p));
    return r;
}

__device__ __forceinline__ uint16_t ld_stream_u16(const uint16_t *p) {
    unsigned short r;
    asm volatile("ld.global.cs.u16 %0, [%1];" : "=h"(r) : "l"(p));
    return r;
}

// ---------------------------------------------------------------------------
// exact block dot: 32 int8 x 32 int8 -> int32, as 8 dp4a
// ---------------------------------------------------------------------------
// (two independent 4-deep dp4a chains, then one add: exact in int32)
__device__ __forceinline__ int block_dot(const uint4 &w0, const uint4 &w1, const uint4 &x0,
                                         const uint4 &x1) {
    int a = __dp4a((int)w0.x, (int)x0.x, 0);
    int b = __dp4a((int)w1.x, (int)x1.x, 0);
    a = __dp4a((int)w0.y, (int)x0.y, a);
    b = __dp4a((int)w1.y, (int)x1.y, b);
    a = __dp4a((int)w0.z, (int)x0.z, a);
    b = __dp4a((int)w1.z, (int)x1.z, b);
    a = __dp4a((int)w0.w, (int)x0.w, a);
    b = __dp4a((int)w1.w, (int)x1.w, b);
    return a + b;
}

}  // namespace q8
