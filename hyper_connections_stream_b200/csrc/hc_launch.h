// hc_launch.h -- internal interface between the C-ABI host layer (hc_api.cu)
// and the kernel translation units (one per storage dtype and kernel kind).
#pragma once

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

// Input-dependent mixing logits on the tensor cores (bf16 H and W).
hc_status launch_mix_logits(const void *H, const void *W, float *z, int64_t T, int n, int64_t d,
                            int P, float eps, const LaunchCtx &ctx, cudaStream_t st);

hc_status launch_selftest_wait(int limit_us, const LaunchCtx &ctx, cudaStream_t st);

hc_status launch_sinkhorn(const float *L, float *out, int64_t T, int n, int K,
                          const LaunchCtx &ctx, cudaStream_t st);

}  // namespace hc
