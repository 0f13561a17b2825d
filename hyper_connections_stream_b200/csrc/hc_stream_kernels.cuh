// hc_stream_kernels.cuh -- register-streaming kernels of the HC step.
//
// One CTA works on one token at a time (tokens blockIdx.x, blockIdx.x + G,
// ... for a grid of G CTAs sized to fill the SMs). Thread c of the CTA owns
// the 16-byte column slices c, c + NT, ... of the token's d axis across all n
// streams, so every global access is a coalesced 128-bit load or store along
// d. Mixing parameters for the next TB tokens are prepared ahead in shared
// memory by lane groups (Sinkhorn / softmax in registers).
//
// KIND_WRITE:  H, y -> H'                    (no reduction, no barrier per token)
// KIND_READ:   H -> x = RMSNorm(a^T H) g
// KIND_FUSED:  H, y -> H', x = RMSNorm(a^T H') g (H' not read back)
// KIND_EXPAND:      e -> H' with every stream a copy of e (p.y holds e)
// KIND_EXPAND_READ: e -> H' as above, x = RMSNorm(a^T H') g (H' not read back)
// KIND_COLLAPSE:    H -> x = a^T H, stored without normalisation
// For the normalising kinds a thread keeps its slice of h in registers until
// the CTA-wide fp64 sum of squares is known (warp shuffles, then one
// shared-memory exchange per token), so each byte crosses HBM once.
#pragma once

#include "hc_device.cuh"

namespace hc {

// Shared memory of the streaming kernels (static size, bounded by n <= 8).
constexpr int kPrepTokens = 32;  // parameter slots prepared per batch (max)

template <int N, typename S, int KIND, int CPT>
__global__ void __launch_bounds__(kStreamMaxThreads)
hc_stream_kernel(StepParams p) {
    constexpr int V = StorageTraits<S>::V;
    constexpr int NN = N * N;
    constexpr bool WRITE = KIND == KIND_WRITE || KIND == KIND_FUSED;  // A, b per token
    constexpr bool READ = KIND != KIND_WRITE && KIND != KIND_EXPAND;  // a per token
    constexpr int TB_MAX = kPrepTokens;

    __shared__ float sA[TB_MAX * NN > 0 ? TB_MAX * NN : 1];
    __shared__ float sb[TB_MAX * N];
    __shared__ float sa[TB_MAX * N];
    __shared__ double sred[2][kStreamMaxThreads / 32];
    __shared__ float swork[kStreamMaxThreads / 32 * kGroupScratch];

    const int tid = threadIdx.x;
    const int NT = blockDim.x;
    const int nwarps = NT >> 5;
    const int64_t nvec = p.d / V;
    const int64_t G = gridDim.x;

    // tokens per parameter batch: a whole number of lane groups per warp
    int TB = nwarps * Group<N>::TPW;
    TB = TB < TB_MAX ? TB : TB_MAX;

    const S *H = static_cast<const S *>(p.H);
    const S *Y = static_cast<const S *>(p.y);
    S *Ho = static_cast<S *>(p.Hout);
    S *X = static_cast<S *>(p.x);

    int parity = 0;
    for (int64_t m0 = 0;; m0 += TB) {
        const int64_t first = blockIdx.x + m0 * G;
        if (first >= p.T) break;
        __syncthreads();  // previous batch's parameters no longer read
        prepare_params<N, WRITE, READ>(p, first, G, TB, sA, sb, sa, swork);
        __syncthreads();

        for (int tt = 0; tt < TB; ++tt) {
            const int64_t t = first + (int64_t)tt * G;
            if (t >= p.T) break;  // uniform over the CTA
            const S *Ht = H + t * N * p.d;
            S *Hot = Ho + t * N * p.d;

            if constexpr (KIND == KIND_EXPAND) {
                for (int64_t c = tid; c < nvec; c += NT) {
                    const int64_t k = c * V;
                    float e[V];
                    load_vec_cs(Y + t * p.d + k, e);
#pragma unroll
                    for (int j = 0; j < N; ++j) store_vec_cs(Hot + j * p.d + k, e);
                }
            } else if constexpr (KIND == KIND_COLLAPSE) {
                S *Xt = X + t * p.d;
                for (int64_t c = tid; c < nvec; c += NT) {
                    const int64_t k = c * V;
                    float h[N][V], acc[V];
#pragma unroll
                    for (int i = 0; i < N; ++i) load_vec_cs(Ht + i * p.d + k, h[i]);
#pragma unroll
                    for (int e = 0; e < V; ++e) acc[e] = -0.0f;
#pragma unroll
                    for (int i = 0; i < N; ++i) {
                        const float ai = sa[tt * N + i];
#pragma unroll
                        for (int e = 0; e < V; ++e) acc[e] = __fmaf_rn(ai, h[i][e], acc[e]);
                    }
                    store_vec_cs(Xt + k, acc);
                }
            } else if constexpr (KIND == KIND_WRITE) {
                for (int64_t c = tid; c < nvec; c += NT) {
                    const int64_t k = c * V;
                    float h[N][V], yv[V];
#pragma unroll
                    for (int i = 0; i < N; ++i) load_vec_cs(Ht + i * p.d + k, h[i]);
                    load_vec_cs(Y + t * p.d + k, yv);
#pragma unroll
                    for (int j = 0; j < N; ++j) {
                        float acc[V];
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
                        store_vec_cs(Hot + j * p.d + k, acc);
                    }
                }
            } else {
                // normalising kinds: phase 1 builds h in registers
                float hs[CPT][V];
                double ss = 0.0;
#pragma unroll
                for (int u = 0; u < CPT; ++u) {
                    const int64_t c = tid + (int64_t)u * NT;
                    if (c < nvec) {
                        const int64_t k = c * V;
#pragma unroll
                        for (int e = 0; e < V; ++e) hs[u][e] = -0.0f;
                        if constexpr (KIND == KIND_EXPAND_READ) {
                            // every stream holds e: store the n copies, mix e
                            float ev[V];
                            load_vec_cs(Y + t * p.d + k, ev);
#pragma unroll
                            for (int j = 0; j < N; ++j) {
                                store_vec_cs(Hot + j * p.d + k, ev);
                                const float aj = sa[tt * N + j];
#pragma unroll
                                for (int e = 0; e < V; ++e) hs[u][e] = __fmaf_rn(aj, ev[e], hs[u][e]);
                            }
                        } else if constexpr (KIND == KIND_FUSED) {
                            float h[N][V];
#pragma unroll
                            for (int i = 0; i < N; ++i) load_vec_cs(Ht + i * p.d + k, h[i]);
                            float yv[V];
                            load_vec_cs(Y + t * p.d + k, yv);
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
                        } else {
                            float h[N][V];
#pragma unroll
                            for (int i = 0; i < N; ++i) load_vec_cs(Ht + i * p.d + k, h[i]);
#pragma unroll
                            for (int i = 0; i < N; ++i) {
                                const float ai = sa[tt * N + i];
#pragma unroll
                                for (int e = 0; e < V; ++e) hs[u][e] = __fmaf_rn(ai, h[i][e], hs[u][e]);
                            }
                        }
#pragma unroll
                        for (int e = 0; e < V; ++e) {
                            const double hv = (double)hs[u][e];
                            ss = __fma_rn(hv, hv, ss);  // hv*hv is exact in fp64
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
                S *Xt = X + t * p.d;
#pragma unroll
                for (int u = 0; u < CPT; ++u) {
                    const int64_t c = tid + (int64_t)u * NT;
                    if (c < nvec) {
                        const int64_t k = c * V;
                        float gv[V], xv[V];
                        load_gain<V>(p.g, k, gv);
#pragma unroll
                        for (int e = 0; e < V; ++e) xv[e] = __fmul_rn(__fmul_rn(hs[u][e], r), gv[e]);
                        store_vec_cs(Xt + k, xv);
                    }
                }
            }
        }
    }
}

// Standalone Sinkhorn projection: each lane group projects one token's n x n
// logits and writes the matrix. Grid-stride over groups of tokens.
template <int N>
__global__ void __launch_bounds__(256)
hc_sinkhorn_kernel(const float *L, float *out, int64_t T, int K) {
    constexpr int NN = N * N, GL = Group<N>::GL, EPL = Group<N>::EPL, TPW = Group<N>::TPW;
    __shared__ float swork[256 / 32 * kGroupScratch];
    const int lane = threadIdx.x & 31;
    const int q = lane & (GL - 1);
    float *wscratch = swork + (threadIdx.x >> 5) * kGroupScratch;
    const int64_t warp_global = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    const int64_t nwarps_global = ((int64_t)gridDim.x * blockDim.x) >> 5;
    for (int64_t t0 = warp_global * TPW; t0 < T; t0 += nwarps_global * TPW) {
        const int64_t t = t0 + lane / GL;
        const bool live = t < T;
        float m[EPL];
#pragma unroll
        for (int r = 0; r < EPL; ++r) {
            const int e = q + GL * r;
            m[r] = (live && e < NN) ? L[t * NN + e] : 0.0f;
        }
        group_sinkhorn<N>(m, wscratch, lane, K);
        if (live) {
#pragma unroll
            for (int r = 0; r < EPL; ++r) {
                const int e = q + GL * r;
                if (e < NN) out[t * NN + e] = m[r];
            }
        }
    }
}

}  // namespace hc
