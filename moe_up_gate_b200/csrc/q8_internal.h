// q8_internal.h -- host-side helpers shared by the libq8 translation units:
// argument validation, the per-thread error detail, launch checks and the
// workspace layout of the routed (MoE) calls.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>
#include <stdio.h>

#include "../../include/q8.h"

namespace q8 {

// Per-thread detail text of the last failure (q8_last_error).
void set_error_detail(const char *fmt, ...);

inline bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
inline bool aligned256(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 255u) == 0; }

#define Q8_FAIL(code, ...)                 \
    do {                                   \
        ::q8::set_error_detail(__VA_ARGS__); \
        return (code);                     \
    } while (0)

#define Q8_REQUIRE(cond, code, ...)        \
    do {                                   \
        if (!(cond)) Q8_FAIL(code, __VA_ARGS__); \
    } while (0)

// After a kernel launch: turn a launch error into Q8_E_CUDA.
inline q8_status launch_status(const char *what) {
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) {
        set_error_detail("%s: %s", what, cudaGetErrorString(e));
        return Q8_E_CUDA;
    }
    return Q8_OK;
}

// Launch with programmatic stream serialization.  The kernel must execute
// griddepcontrol.wait before it reads anything an earlier kernel writes
// (and before it writes anything an earlier kernel reads).
template <typename... KArgs, typename... Args>
inline q8_status launch_pdl(const char *what, void (*kern)(KArgs...), dim3 grid, dim3 block,
                            size_t smem, cudaStream_t s, Args... args) {
    cudaLaunchConfig_t cfg{};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    cudaError_t e = cudaLaunchKernelEx(&cfg, kern, args...);
    if (e != cudaSuccess) {
        set_error_detail("%s: launch: %s", what, cudaGetErrorString(e));
        return Q8_E_CUDA;
    }
    return Q8_OK;
}

// Validate a weight view.  need_single: n_mat must be 1.
q8_status check_tensor(const q8_tensor *W, const char *name, bool need_single);

// ---------------------------------------------------------------------------
// Routed-call workspace: int32 words.
//   [0] error flags  [1] number of experts in the dp4a list  [2] number in the
//   tensor-core list  [3] pairs  [4] [5] the fused layer kernel's grid-barrier
//   arrival counter (64 bits)  [6] [7] unused, then count[E], offset[E+1],
//   list_small[E], list_big[E], pairs[P] (pair index p = t * n_used + s,
//   sorted by expert, then p).
// No grouping writes words 4-7, so the barrier words keep their place and
// their zero whatever the shape of the calls that share a workspace.
// ---------------------------------------------------------------------------
enum : int {
    WS_ERR = 0,
    WS_N_SMALL = 1,
    WS_N_BIG = 2,
    WS_N_PAIRS = 3,
    WS_BAR = 4,
    WS_HEADER = 8
};
enum : int { ERR_ID_RANGE = 1, ERR_ID_REPEAT = 2 };

struct GroupLayout {
    int64_t count, offset, list_small, list_big, pairs, words;
};

inline GroupLayout group_layout(int64_t n_pairs, int64_t n_mat) {
    GroupLayout L;
    L.count = WS_HEADER;
    L.offset = L.count + n_mat;
    L.list_small = L.offset + n_mat + 1;
    L.list_big = L.list_small + n_mat;
    L.pairs = L.list_big + n_mat;
    L.words = L.pairs + n_pairs;
    return L;
}

inline size_t round_up(size_t v, size_t a) { return (v + a - 1) / a * a; }

inline size_t group_bytes(int64_t n_pairs, int64_t n_mat) {
    return round_up((size_t)group_layout(n_pairs, n_mat).words * 4, 256);
}

// Whether a kernel has been given the full shared-memory opt-in on a device
// (q8_quant.cu keeps the registry, guarded by a mutex).
bool smem_opted_in(const void *kernel, int device);
void set_smem_opted_in(const void *kernel, int device);

// Number of SMs of the current device (cached per device).
int num_sms();

// Quantize rows (q8_quant.cu): scales to d[row * ld_d + b].  weights: the
// output is packed weights (the next kernel may not start before it ends).
q8_status launch_quantize(const float *x, int64_t n_rows, int64_t k, int8_t *qs, uint16_t *d,
                          int64_t ld_d, cudaStream_t s, bool weights = false);

// Streaming matmuls (q8_matmul.cu).  Activations are Q8_0 (aq, ad) or fp32
// (af, quantized by the Q8_0 rule as they are staged).
q8_status launch_matmul_routed(const q8_tensor *W, const int8_t *aq, const uint16_t *ad,
                               const float *af, int a_per_slot, int64_t n_tok, int32_t n_used,
                               float *y, const int32_t *ws, cudaStream_t s);
q8_status launch_matmul_dense(const q8_tensor *W, const int8_t *aq, const uint16_t *ad,
                              const float *af, int64_t n_tok, float *y, cudaStream_t s);
q8_status launch_matmul_routed_ids(const q8_tensor *W, const int8_t *aq, const uint16_t *ad,
                                   const float *af, int a_per_slot, int64_t n_tok,
                                   int32_t n_used, const int32_t *ids, float *y,
                                   int32_t *err_out, cudaStream_t s);

// Rows per compute pass (the kernels' NT; a pass over fewer rows runs a
// narrower variant at run time) and rows staged in shared memory at once
// (every row of an expert where possible: restaging per tile costs a memory
// latency each time).  An expert has at most n_tok rows.
struct RowPlan {
    int64_t nt_rows, x_rows;
};
inline RowPlan routed_rows(int64_t n_tok, int64_t n_used, int64_t n_mat) {
    (void)n_used;
    (void)n_mat;
    RowPlan r;
    r.nt_rows = n_tok;
    r.x_rows = n_tok < 16 ? n_tok : 16;
    return r;
}
inline RowPlan dense_rows(int64_t n_tok) { return RowPlan{n_tok, n_tok < 16 ? n_tok : 16}; }

// Batches small enough for the grouping to be built inside each CTA.
constexpr int64_t kCtaGroupMaxPairs = Q8_SMALL_BATCH_PAIRS;
constexpr int64_t kCtaGroupMaxMats = Q8_SMALL_BATCH_MATS;

// Wait-timeout flags latched by the streaming kernels of each file.
// The fused MoE layer kernel (q8_layer.cu) for small routed batches.
constexpr int64_t kLayerMaxPairs = 32;
bool layer_eligible(const q8_tensor *up_gate, const q8_tensor *down, int64_t n_tok,
                    int32_t n_used);
q8_status launch_layer(const q8_tensor *up_gate, const q8_tensor *down, const float *x,
                       int64_t n_tok, const int32_t *ids, const float *route_w, int32_t n_used,
                       float *out, float *h, unsigned *bar, int32_t *err_out, cudaStream_t s);
q8_status read_wait_errors_layer(int *flags);

q8_status read_wait_errors_matmul(int *flags);
q8_status read_wait_errors_moe(int *flags);
q8_status read_wait_errors_tc(int *flags);
// Zero the wait-timeout flag of each file on the current device.
q8_status clear_wait_errors_layer();
q8_status clear_wait_errors_matmul();
q8_status clear_wait_errors_moe();
q8_status clear_wait_errors_tc();

// Tensor-core path (q8_tc.cu) for experts with at least kTcMinPairs routed
// rows: whether a weight view can take it, and the launch over the
// tensor-core list of a grouping workspace.  From 4 rows on, a 16-column MMA
// pass (padded) costs less per weight byte than the dp4a kernel: the
// 128-expert layer at 256 tokens ran 1.3x faster than with a 16-row
// threshold.
constexpr int kTcMinPairs = 4;
// Dense calls (one matrix) with kTcMinDense..kTcMaxDense activation rows go
// to the tensor cores too (one pass over the weights): launch_tc with
// ws == nullptr.  (4 rows, the routed experts' line, measured no faster
// for the dense 8-row up/gate of fp32 activations: their quantization in the
// gathering warps then costs what the dp4a kernel saves.)
constexpr int kTcMinDense = 16;
constexpr int kTcMaxDense = 32;
bool tc_eligible(const q8_tensor *W, bool upgate);
q8_status launch_tc(const q8_tensor *W, bool upgate, const int8_t *aq, const uint16_t *ad,
                    const float *af, int a_per_slot, int64_t n_tok, int32_t n_used, float *out,
                    const int32_t *ws, cudaStream_t s);

// Launch the expert-grouping kernel (q8_moe.cu).  big_threshold: experts with
// at least this many pairs go to the tensor-core list.
q8_status launch_group(const int32_t *ids, int64_t n_tok, int32_t n_used, int64_t n_mat,
                       int32_t big_threshold, int32_t *ws, cudaStream_t s);

}  // namespace q8
