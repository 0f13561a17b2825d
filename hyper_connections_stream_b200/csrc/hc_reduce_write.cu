// hc_reduce_write.cu -- the write mix fused with the tensor-parallel
// all-reduce of the block output, then the next layer's read, in one pass.
//
// Under tensor parallelism (Hy4-preview model techniques map, the "inference
// kernel" row: Hy4's kernels are fused and the model is served split over
// eight GPUs) each of R ranks ends a block with a partial y_r of the block's
// output and holds a replica of the streams H. Here every rank reads all R
// partials -- its own from HBM, the others' from peer memory over NVLink --
// sums them, and applies the write mix of the glossary entry
// "Hyper-connections (mHC)" and the next block's read + pre-norm RMSNorm:
//   y    = rnd_s( ((y_0 + y_1) + y_2) + ... + y_{R-1} )  fp32, rank order
//   H'_j = sum_i A[i][j] H_i + b_j y,   x = RMSNorm(sum_j a_j H'_j) * g
// The fixed order makes y, and therefore H' and x, bit-identical on every
// rank, so the replicas of H stay equal without another exchange. y never
// makes a round trip through HBM unless the caller asks for it.
//
// Two forms share the kernel. One-shot (hc_reduce_write_then_read): every
// rank reduces every token and writes its own replica of H' and x. Reduce-
// scatter (hc_reduce_scatter_write_then_read): the streams are sharded by
// token over the ranks; a rank reduces the partials' rows of its own tokens
// only, writes its shard of H', and stores that shard's x_next into every
// rank's x buffer (the all-gather, as plain stores to peer memory).
//
// Peer memory is read and written with plain loads and stores only (bulk
// copies, never multicast, read this GPU's own memory), and no kernel ever
// waits on another rank: the caller orders each
// partial's writes before the call, and every later read of x or overwrite
// of a partial after every rank's call (the host layer does this with two
// barriers). With buffers of one GPU it is the same computation over all
// ranks' data, one launch per rank.
//
// Two kernel families, as for the step: the pipelined one (hc_pipe_kernel,
// KIND_REDUCE: bulk copies of the stream rows and of the local partial rows
// into shared-memory rings, warp-specialised) for large calls, and the
// register-streaming one below for decode-sized calls and shapes whose ring
// does not fit: one CTA per token at a time (grid-stride), threads own
// 16-byte column slices, and h stays in registers until the CTA's fp64 sum
// of squares is known.
#include "hc_launch.h"

namespace hc {

namespace {

constexpr int kRwPrep = 32;  // parameter slots per batch (max)

template <typename S> struct RwRound;
template <> struct RwRound<float> {
    static __device__ __forceinline__ void apply(float (&)[4]) {}
};
template <> struct RwRound<__nv_bfloat16> {
    static __device__ __forceinline__ void apply(float (&v)[8]) {
#pragma unroll
        for (int e = 0; e < 8; e += 2) widen_bf16x2(pack_bf16x2_rn(v[e], v[e + 1]), v[e], v[e + 1]);
    }
};

template <int N, typename S, int CPT>
__global__ void __launch_bounds__(kStreamMaxThreads)
hc_reduce_step_kernel(ReduceWriteArgs ra) {
    constexpr int V = StorageTraits<S>::V;
    constexpr int NN = N * N;
    const StepParams &p = ra.f;
    __shared__ float sA[kRwPrep * NN], sb[kRwPrep * N], sa[kRwPrep * N];
    __shared__ double sred[2][kStreamMaxThreads / 32];
    __shared__ float swork[kStreamMaxThreads / 32 * kGroupScratch];

    const int tid = threadIdx.x;
    const int NT = blockDim.x;
    const int nwarps = NT >> 5;
    const int64_t nvec = p.d / V;
    const int64_t G = gridDim.x;
    int TB = nwarps * Group<N>::TPW;
    TB = TB < kRwPrep ? TB : kRwPrep;
    const int R = ra.R;

    const S *H = static_cast<const S *>(p.H);
    S *Ho = static_cast<S *>(p.Hout);
    S *Yo = static_cast<S *>(ra.y_out);

    int parity = 0;
    for (int64_t m0 = 0;; m0 += TB) {
        const int64_t first = blockIdx.x + m0 * G;
        if (first >= p.T) break;
        __syncthreads();  // previous batch's parameters no longer read
        prepare_params<N, true, true>(p, first, G, TB, sA, sb, sa, swork);
        __syncthreads();
        for (int tt = 0; tt < TB; ++tt) {
            const int64_t t = first + (int64_t)tt * G;
            if (t >= p.T) break;  // uniform over the CTA
            const S *Ht = H + t * N * p.d;
            S *Hot = Ho + t * N * p.d;
            const int64_t tg = ra.t0 + t;  // row of the partials and of x
            float hs[CPT][V];
            double ss = 0.0;
#pragma unroll
            for (int u = 0; u < CPT; ++u) {
                const int64_t c = tid + (int64_t)u * NT;
                if (c < nvec) {
                    const int64_t k = c * V;
                    float h[N][V], yv[V];
#pragma unroll
                    for (int i = 0; i < N; ++i) load_vec_cs(Ht + i * p.d + k, h[i]);
                    // the all-reduce: partials added in rank order, one rounding
                    load_vec_cs(static_cast<const S *>(ra.parts[0]) + tg * p.d + k, yv);
#pragma unroll
                    for (int r = 1; r < kMaxRanks; ++r) {
                        if (r < R) {
                            float pv[V];
                            load_vec_cs(static_cast<const S *>(ra.parts[r]) + tg * p.d + k, pv);
#pragma unroll
                            for (int e = 0; e < V; ++e) yv[e] = __fadd_rn(yv[e], pv[e]);
                        }
                    }
                    if (Yo) {
                        float stored[V];
                        store_vec_cs(Yo + t * p.d + k, yv, stored);
#pragma unroll
                        for (int e = 0; e < V; ++e) yv[e] = stored[e];
                    } else {
                        RwRound<S>::apply(yv);
                    }
                    // write mix and read mix, exactly as the fused step
#pragma unroll
                    for (int e = 0; e < V; ++e) hs[u][e] = -0.0f;
#pragma unroll
                    for (int j = 0; j < N; ++j) {
                        float acc[V], stored[V];
#pragma unroll
                        for (int e = 0; e < V; ++e) acc[e] = -0.0f;
#pragma unroll
                        for (int i = 0; i < N; ++i) {
                            const float aij = sA[tt * NN + i * N + j];
#pragma unroll
                            for (int e = 0; e < V; ++e) acc[e] = __fmaf_rn(aij, h[i][e], acc[e]);
                        }
                        const float bj = sb[tt * N + j];
#pragma unroll
                        for (int e = 0; e < V; ++e) acc[e] = __fmaf_rn(bj, yv[e], acc[e]);
                        store_vec_cs(Hot + j * p.d + k, acc, stored);
                        const float aj = sa[tt * N + j];
#pragma unroll
                        for (int e = 0; e < V; ++e) hs[u][e] = __fmaf_rn(aj, stored[e], hs[u][e]);
                    }
#pragma unroll
                    for (int e = 0; e < V; ++e) {
                        const double hv = (double)hs[u][e];
                        ss = __fma_rn(hv, hv, ss);
                    }
                }
            }
            // CTA-wide sum of squares: warp tree, then warps in index order
#pragma unroll
            for (int off = 16; off > 0; off >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, off);
            if ((tid & 31) == 0) sred[parity][tid >> 5] = ss;
            __syncthreads();
            double tot = 0.0;
            for (int w = 0; w < nwarps; ++w) tot += sred[parity][w];
            parity ^= 1;
            const float r = __double2float_rn(1.0 / sqrt(tot / (double)p.d + (double)p.eps));
#pragma unroll
            for (int u = 0; u < CPT; ++u) {
                const int64_t c = tid + (int64_t)u * NT;
                if (c < nvec) {
                    const int64_t k = c * V;
                    float gv[V], xv[V];
                    load_gain<V>(p.g, k, gv);
#pragma unroll
                    for (int e = 0; e < V; ++e) xv[e] = __fmul_rn(__fmul_rn(hs[u][e], r), gv[e]);
                    // x_next to every destination (the all-gather of the
                    // reduce-scatter form: peers' buffers take plain stores)
                    store_vec_cs(static_cast<S *>(ra.xs[0]) + tg * p.d + k, xv);
#pragma unroll
                    for (int q = 1; q < kMaxRanks; ++q)
                        if (q < ra.nx) store_vec_cs(static_cast<S *>(ra.xs[q]) + tg * p.d + k, xv);
                }
            }
        }
    }
}

// Threads per CTA and slices per thread for a row of nvec 16-byte slices:
// the least idle slices, then the fewest slices per thread, among CTAs of at
// most 256 threads where one exists (two CTAs per SM then fit the register
// file, so one CTA's loads overlap the other's per-token reduction), else up
// to 512.
void rw_shape(int64_t nvec, int &NT, int &CPT) {
    static const int cpts[] = {1, 2, 4, 8};
    NT = 0;
    CPT = 8;
    for (int cap : {256, kStreamMaxThreads}) {
        int64_t best = INT64_MAX;
        for (int cpt : cpts) {
            int64_t nt = (nvec + cpt - 1) / cpt;
            nt = (nt + 31) / 32 * 32;
            if (nt > cap) continue;
            if (nt < 64 && cpt > 1) continue;
            const int64_t waste = nt * cpt - nvec;
            if (waste < best) {
                best = waste;
                NT = (int)nt;
                CPT = cpt;
            }
        }
        if (NT) return;
    }
}

template <int N, typename S, int CPT>
hc_status rw_launch_cpt(const ReduceWriteArgs &ra, int NT, const LaunchCtx &ctx, cudaStream_t st) {
    auto kern = hc_reduce_step_kernel<N, S, CPT>;
    int per_sm = 0;
    cudaError_t e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, NT, 0);
    if (e != cudaSuccess) return set_error(HC_ERR_CUDA, "occupancy query: %s", cudaGetErrorString(e));
    if (per_sm < 1) per_sm = 1;
    int64_t grid = (int64_t)ctx.sms * per_sm;
    if (grid > ra.f.T) grid = ra.f.T;
    kern<<<(unsigned)grid, NT, 0, st>>>(ra);
    e = cudaGetLastError();
    if (e != cudaSuccess) return set_error(HC_ERR_CUDA, "hc_reduce_step_kernel launch: %s", cudaGetErrorString(e));
    return HC_OK;
}

template <int N, typename S>
hc_status rw_launch_n(const ReduceWriteArgs &ra, const LaunchCtx &ctx, cudaStream_t st) {
    int NT = 0, CPT = 1;
    rw_shape(ra.f.d / StorageTraits<S>::V, NT, CPT);
    if (NT == 0) return set_error(HC_ERR_UNSUPPORTED, "no launch shape for d = %lld", (long long)ra.f.d);
    switch (CPT) {
        case 1: return rw_launch_cpt<N, S, 1>(ra, NT, ctx, st);
        case 2: return rw_launch_cpt<N, S, 2>(ra, NT, ctx, st);
        case 4: return rw_launch_cpt<N, S, 4>(ra, NT, ctx, st);
        default: return rw_launch_cpt<N, S, 8>(ra, NT, ctx, st);
    }
}

template <typename S>
hc_status rw_dispatch(const ReduceWriteArgs &ra, const LaunchCtx &ctx, cudaStream_t st) {
    switch (ra.n) {
        case 1: return rw_launch_n<1, S>(ra, ctx, st);
        case 2: return rw_launch_n<2, S>(ra, ctx, st);
        case 3: return rw_launch_n<3, S>(ra, ctx, st);
        case 4: return rw_launch_n<4, S>(ra, ctx, st);
        case 5: return rw_launch_n<5, S>(ra, ctx, st);
        case 6: return rw_launch_n<6, S>(ra, ctx, st);
        case 7: return rw_launch_n<7, S>(ra, ctx, st);
        default: return rw_launch_n<8, S>(ra, ctx, st);
    }
}

}  // namespace

hc_status launch_reduce_write(const ReduceWriteArgs &ra, hc_dtype dt, const LaunchCtx &ctx,
                              cudaStream_t st) {
    // Decode-sized calls (under ~64 MiB of stream traffic) skip the pipeline's
    // set-up, as the step kinds do; hc_set_path forces either family.
    const int64_t es = dt == HC_BF16 ? 2 : 4;
    const bool small = ra.f.T * (int64_t)ra.n * ra.f.d * es * 2 < (int64_t(64) << 20);
    if (ctx.path == 1 || (ctx.path == 0 && !small)) {
        // partials in this GPU's own memory are staged by bulk copies; any
        // other (a peer's memory, or memory the runtime cannot place) takes
        // plain loads
        bool local[kMaxRanks] = {};
        for (int r = 0; r < ra.R; ++r) {
            cudaPointerAttributes at{};
            const cudaError_t e = cudaPointerGetAttributes(&at, ra.parts[r]);
            if (e != cudaSuccess) {
                (void)cudaGetLastError();  // not a device pointer the runtime knows: plain loads
                continue;
            }
            local[r] = at.type == cudaMemoryTypeDevice && at.device == ctx.device;
        }
        bool fits = false;
        const hc_status s = dt == HC_BF16 ? launch_reduce_pipe<__nv_bfloat16>(ra, local, ctx, st, &fits)
                                          : launch_reduce_pipe<float>(ra, local, ctx, st, &fits);
        if (s != HC_OK || fits) return s;
        if (ctx.path == 1)
            return set_error(HC_ERR_UNSUPPORTED, "pipelined kernels do not cover d = %lld with R = %d here",
                             (long long)ra.f.d, ra.R);
    }
    return dt == HC_BF16 ? rw_dispatch<__nv_bfloat16>(ra, ctx, st) : rw_dispatch<float>(ra, ctx, st);
}

}  // namespace hc
