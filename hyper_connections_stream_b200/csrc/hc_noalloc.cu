// hc_noalloc.cu -- hc_write_then_read_backward_noalloc: the backward pass with
// its gain-gradient scratch in a file-scope device array instead of a caller
// workspace, so a call allocates nothing and needs no workspace argument.
//
// Who needs it: callers that may not allocate device memory at the point of
// the call -- runtimes that reserve all of a GPU's memory up front in their
// own pool and hand kernels no spare buffer, and latency-critical loops where
// a cudaMalloc (which can synchronise the whole device) is not acceptable.
//
// The scratch is one array per device (statically sized; calls that would
// need more are rejected with HC_ERR_UNSUPPORTED before any launch). In host
// code the array's name is only a stand-in for the device copy, so its device
// address is looked up once per device, with that device current, by
// cudaGetSymbolAddress, and cached. Nothing in it has to start at zero: the
// step kernel writes every partial row it later reduces. Every call on a
// device shares the array; calls whose executions overlap race on it.
#include <atomic>

#include "hc_launch.h"

namespace {

constexpr size_t kNoAllocScratchBytes = size_t(16) << 20;  // 16 MiB
static __device__ __align__(256) unsigned char g_hc_bw_scratch[kNoAllocScratchBytes];

constexpr int kMaxDevices = 64;
std::atomic<void *> g_scratch_addr[kMaxDevices];

hc_status noalloc_fail(hc_status st, const char *msg) { return hc::set_error(st, "%s", msg); }

}  // namespace

extern "C" {

HC_API hc_status hc_write_then_read_backward_noalloc(
    const void *H, const void *y, hc_dtype dt, int64_t T, int n, int64_t d, hc_mix_mode mm,
    const float *A, int64_t A_tok_stride, int K, const float *b, int64_t b_tok_stride,
    hc_read_mode rm, const float *a, int64_t a_tok_stride, const float *g, float eps,
    const void *dHout, const void *dx, void *dH, void *dy, float *dA, float *db, float *da,
    float *dg, hc_stream stream) {
    void *scratch = nullptr;
    size_t scratch_bytes = 0;
    if (dg && T > 0) {
        int dev = 0;
        if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices)
            return noalloc_fail(HC_ERR_CUDA, "hc_write_then_read_backward_noalloc: no current device");
        scratch = g_scratch_addr[dev].load(std::memory_order_acquire);
        if (!scratch) {
            cudaError_t e = cudaGetSymbolAddress(&scratch, g_hc_bw_scratch);
            if (e != cudaSuccess)
                return hc::set_error(HC_ERR_CUDA,
                                     "hc_write_then_read_backward_noalloc: cudaGetSymbolAddress(scratch): %s",
                                     cudaGetErrorString(e));
            g_scratch_addr[dev].store(scratch, std::memory_order_release);
        }
        // need == 0 flags arguments or a launch plan the backward rejects: the
        // call below then reports that status and text itself (its checks run
        // before anything touches the scratch)
        const size_t need = hc_write_then_read_backward_workspace_bytes(dt, T, n, d);
        if (need > kNoAllocScratchBytes)
            return hc::set_error(HC_ERR_UNSUPPORTED,
                                 "hc_write_then_read_backward_noalloc: the gain gradient needs %zu bytes "
                                 "of partials, more than the 16 MiB static scratch (use "
                                 "hc_write_then_read_backward with a workspace)",
                                 need);
        scratch_bytes = kNoAllocScratchBytes;
    }
    return hc_write_then_read_backward(H, y, dt, T, n, d, mm, A, A_tok_stride, K, b, b_tok_stride,
                                       rm, a, a_tok_stride, g, eps, dHout, dx, dH, dy, dA, db, da,
                                       dg, scratch, scratch_bytes, stream);
}

}  // extern "C"
