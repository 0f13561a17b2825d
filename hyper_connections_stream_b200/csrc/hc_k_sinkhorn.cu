// Standalone Sinkhorn projection launcher (hc_sinkhorn).
#include "hc_launch.h"
#include "hc_stream_kernels.cuh"

namespace hc {

hc_status launch_sinkhorn(const float *L, float *out, int64_t T, int n, int K,
                          const LaunchCtx &ctx, cudaStream_t st) {
    const int threads = 256;
    int tpw = 1;
    switch (n) {
        case 1: tpw = Group<1>::TPW; break;
        case 2: tpw = Group<2>::TPW; break;
        case 3: tpw = Group<3>::TPW; break;
        case 4: tpw = Group<4>::TPW; break;
        default: tpw = 1; break;
    }
    const int64_t tokens_per_cta = (int64_t)(threads / 32) * tpw;
    int64_t grid = (T + tokens_per_cta - 1) / tokens_per_cta;
    const int64_t gmax = (int64_t)ctx.sms * 8;
    if (grid > gmax) grid = gmax;
    const unsigned gr = (unsigned)grid;
    switch (n) {
        case 1: hc_sinkhorn_kernel<1><<<gr, threads, 0, st>>>(L, out, T, K); break;
        case 2: hc_sinkhorn_kernel<2><<<gr, threads, 0, st>>>(L, out, T, K); break;
        case 3: hc_sinkhorn_kernel<3><<<gr, threads, 0, st>>>(L, out, T, K); break;
        case 4: hc_sinkhorn_kernel<4><<<gr, threads, 0, st>>>(L, out, T, K); break;
        case 5: hc_sinkhorn_kernel<5><<<gr, threads, 0, st>>>(L, out, T, K); break;
        case 6: hc_sinkhorn_kernel<6><<<gr, threads, 0, st>>>(L, out, T, K); break;
        case 7: hc_sinkhorn_kernel<7><<<gr, threads, 0, st>>>(L, out, T, K); break;
        default: hc_sinkhorn_kernel<8><<<gr, threads, 0, st>>>(L, out, T, K); break;
    }
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return set_error(HC_ERR_CUDA, "hc_sinkhorn_kernel launch: %s", cudaGetErrorString(e));
    return HC_OK;
}

}  // namespace hc
