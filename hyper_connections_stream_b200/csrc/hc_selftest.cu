// Self-test of the bounded-wait mechanism: one thread waits on a shared-memory
// mbarrier that nothing ever arrives at, with a caller-given limit. The wait
// must give up, OR FAULT_SELFTEST into the device fault word and let the
// kernel return normally. No copy is in flight and nothing traps, so the
// context stays usable; the host reads the word with hc_device_fault().
#include "hc_launch.h"
#include "hc_sync.cuh"

namespace hc {

__global__ void __launch_bounds__(32) hc_selftest_wait_kernel(int *fault, uint64_t limit_ns) {
    __shared__ uint64_t bar;
    if (threadIdx.x != 0) return;
    mbar_init(&bar, 1);
    fence_barrier_init();
    const uint64_t t0 = global_timer_ns();
    for (uint32_t it = 0;; ++it) {
        if (mbar_try_wait(&bar, 0)) return;  // never completes: nothing arrives
        if ((it & 15u) == 15u && global_timer_ns() - t0 > limit_ns) {
            atomicOr(fault, FAULT_SELFTEST);
            return;
        }
    }
}

hc_status launch_selftest_wait(int limit_us, const LaunchCtx &ctx, cudaStream_t st) {
    hc_selftest_wait_kernel<<<1, 32, 0, st>>>(ctx.fault, (uint64_t)limit_us * 1000ull);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess)
        return set_error(HC_ERR_CUDA, "hc_selftest_wait_kernel launch: %s", cudaGetErrorString(e));
    return HC_OK;
}

}  // namespace hc
