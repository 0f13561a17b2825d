// hc_launch.h -- internal interface between the C-ABI host layer (hc_api.cu)
// and the kernel translation units (one per storage dtype and kernel kind).
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>

#include "hc_api.h"
#include "hc_device.cuh"

namespace hc {

constexpr int kSmemLimitLogits = 232448;  // 227 KB opt-in dynamic shared memory per CTA

struct LaunchCtx {
    int device;  // current device ordinal
    int sms;     // SMs of the current device
    int *fault;  // device fault word of the current device
    int path;    // hc_path: 0 auto, 1 pipelined, 2 register-streaming
};

// Record the calling thread's error text and return st.
hc_status set_error(hc_status st, const char *fmt, ...);

// Launch one step kind (KIND_READ / KIND_WRITE / KIND_FUSED) for n streams.
template <typename S, int KIND>
hc_status launch_kind(int n, const StepParams &p, const LaunchCtx &ctx, cudaStream_t st);
// The kernel family launch_kind would take for p: 1 pipelined, 2 register-streaming.
template <typename S, int KIND>
int step_path(int n, const StepParams &p, const LaunchCtx &ctx);

// 2-D bf16 TMA tensor map over a row-major [outer][inner] array: 128-byte
// swizzle, zero fill out of bounds, box of box_outer rows x box_inner elements.
hc_status make_tma_map_bf16(CUtensorMap *map, const void *base, uint64_t inner, uint64_t outer,
                            uint32_t box_inner, uint32_t box_outer);

// Input-dependent mixing logits on the tensor cores (bf16 H and W).
hc_status launch_mix_logits(const void *H, const void *W, float *z, int64_t T, int n, int64_t d,
                            int P, float eps, const LaunchCtx &ctx, cudaStream_t st);

// The block's output projection fused with the write mix (bf16):
// y = X Wo^T on the tensor cores, H'_j = sum_i A[i][j] H_i + b_j y.
struct LinearWriteArgs {
    const void *X, *Wo, *H;
    void *Hout, *y;  // y may be null
    int64_t T, d, k;
    int n;
    const float *A;
    int64_t A_s;
    const float *b;
    int64_t b_s;
};
hc_status launch_linear_write(const LinearWriteArgs &a, const LaunchCtx &ctx, cudaStream_t st);

// Backward pass of the fused step (see hc_write_then_read_backward).
struct BackwardArgs {
    StepParams f;  // forward inputs: H, y, A, b, a, g, eps, K, modes, T, d
    int n;
    hc_dtype dt;
    const void *dHout;  // [T][n][d] or null
    const void *dx;     // [T][d]
    void *dH;           // [T][n][d]
    void *dy;           // [T][d]
    float *dA, *db, *da, *dg;
    void *workspace;
    size_t workspace_bytes;
};
// Workspace the backward needs for the gain gradient on the current device.
hc_status backward_workspace_bytes(int n, hc_dtype dt, int64_t T, int64_t d, const LaunchCtx &ctx,
                                   size_t *bytes);
hc_status launch_backward(const BackwardArgs &a, const LaunchCtx &ctx, cudaStream_t st);

// The write mix fused with the tensor-parallel all-reduce of y, then the
// next layer's read (see hc_reduce_write_then_read).
constexpr int kMaxRanks = 8;
struct ReduceWriteArgs {
    StepParams f;                  // H, Hout, params, T (tokens of this call), d (f.y, f.x unused)
    const void *parts[kMaxRanks];  // the ranks' partial y, in rank order
    int R;
    int n;
    void *y_out;                   // reduced y [T][d] (this call's tokens), or null
    int64_t t0;                    // row of the partials and of x for this call's token 0
    void *xs[kMaxRanks];           // x_next destinations (rows t0 .. t0 + T - 1 of each)
    int nx;
};
hc_status launch_reduce_write(const ReduceWriteArgs &ra, hc_dtype dt, const LaunchCtx &ctx,
                              cudaStream_t st);
// Its pipelined (TMA-fed) form; local[r] marks partials in this GPU's memory
// (staged by bulk copies; the others are read with plain loads). Launches
// nothing and sets *fits = false when the ring does not fit shared memory.
template <typename S>
hc_status launch_reduce_pipe(const ReduceWriteArgs &ra, const bool *local, const LaunchCtx &ctx,
                             cudaStream_t st, bool *fits);

hc_status launch_selftest_wait(int limit_us, const LaunchCtx &ctx, cudaStream_t st);

hc_status launch_sinkhorn(const float *L, float *out, int64_t T, int n, int K,
                          const LaunchCtx &ctx, cudaStream_t st);

}  // namespace hc
