// hc_pipe_kernels.cuh -- warp-specialised, TMA-fed kernels of the HC step.
//
// One persistent CTA per SM (tokens blockIdx.x, blockIdx.x + G, ...), 512
// threads in three roles:
//   warp 0      producer: one lane streams each token's n stream rows (and y)
//               tile by tile into a ring of shared-memory stages with plain
//               bulk copies (cp.async.bulk, this GPU's own memory, no
//               multicast), completing on the stage's "full" mbarrier;
//   warp 1      parameters: lane groups compute the per-token Sinkhorn
//               projection / read softmax ahead of use into a slot ring;
//   warps 2-15  two consumer groups of 7 warps; each group owns whole tokens
//               (alternating), reads the stages, writes H' with coalesced
//               128-bit stores, keeps its slice of h in registers, reduces the
//               fp64 sum of squares across its warps, then stores x.
// The producer runs up to `stages` tiles ahead, so HBM always has tens of
// kilobytes per SM in flight while the consumers compute, reduce and store.
//
// Every wait is bounded (hc_sync.cuh): on time-out the CTA records a fault
// code, stops issuing, drains the copies it issued and exits.
#pragma once

#include "hc_device.cuh"
#include "hc_sync.cuh"

namespace hc {

constexpr int kPipeThreads = 512;
constexpr int kPipeGroups = 2;
constexpr int kPipeGroupWarps = 7;
constexpr int kPipeGroupThreads = kPipeGroupWarps * 32;
constexpr int kParamSlots = 16;
constexpr int kMaxStages = 32;
constexpr int kSmemLimit = 232448;  // 227 KB opt-in dynamic shared memory per CTA

struct PipeShape {
    int stages;       // ring depth
    int tile;         // elements of d per tile (= kPipeGroupThreads * V)
    int ntile;        // tiles per token
    int stage_bytes;  // bytes of one stage
};

// Bytes of everything in shared memory other than the ring.
__host__ __device__ constexpr int pipe_fixed_bytes(int n, int stages) {
    return stages * 16                                 // full + empty barriers
           + kParamSlots * 16                          // param full + empty
           + kPipeGroups * 8                           // group reduction barriers
           + kParamSlots * (n * n + 2 * n) * 4         // parameter slots
           + kPipeGroups * 2 * kPipeGroupWarps * 8     // reduction partials
           + 16;                                       // abort flag (padded)
}

template <typename S> struct SmemVec;
template <> struct SmemVec<float> {
    static __device__ __forceinline__ void load(const unsigned char *p, float (&v)[4]) {
        const float4 q = *reinterpret_cast<const float4 *>(p);
        v[0] = q.x; v[1] = q.y; v[2] = q.z; v[3] = q.w;
    }
};
template <> struct SmemVec<__nv_bfloat16> {
    static __device__ __forceinline__ void load(const unsigned char *p, float (&v)[8]) {
        const uint4 q = *reinterpret_cast<const uint4 *>(p);
        widen_bf16x2(q.x, v[0], v[1]);
        widen_bf16x2(q.y, v[2], v[3]);
        widen_bf16x2(q.z, v[4], v[5]);
        widen_bf16x2(q.w, v[6], v[7]);
    }
};

template <int N, typename S, int KIND, int HT>
__global__ void __launch_bounds__(kPipeThreads, 1)
hc_pipe_kernel(StepParams p, PipeShape sh, int *fault) {
    constexpr int V = StorageTraits<S>::V;
    constexpr int NN = N * N;
    constexpr bool WRITE = KIND != KIND_READ;
    constexpr bool READ = KIND != KIND_WRITE;
    constexpr int ROWS = WRITE ? N + 1 : N;
    constexpr int PSTRIDE = NN + 2 * N;  // A | b | a
    constexpr int GW = kPipeGroupWarps;

    extern __shared__ __align__(128) unsigned char smem[];
    unsigned char *ring = smem;
    uint64_t *full = reinterpret_cast<uint64_t *>(smem + (size_t)sh.stages * sh.stage_bytes);
    uint64_t *empty = full + sh.stages;
    uint64_t *pfull = empty + sh.stages;
    uint64_t *pempty = pfull + kParamSlots;
    uint64_t *redbar = pempty + kParamSlots;
    float *params = reinterpret_cast<float *>(redbar + kPipeGroups);
    double *sred = reinterpret_cast<double *>(params + kParamSlots * PSTRIDE);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(sred + kPipeGroups * 2 * GW);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    if (threadIdx.x == 0) {
        for (int s = 0; s < sh.stages; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], GW);
        }
        for (int s = 0; s < kParamSlots; ++s) {
            mbar_init(&pfull[s], 1);
            mbar_init(&pempty[s], GW);
        }
        for (int g = 0; g < kPipeGroups; ++g) mbar_init(&redbar[g], GW);
        *abort_flag = 0;
        fence_barrier_init();
    }
    __syncthreads();

    const int64_t G = gridDim.x;
    const int64_t d = p.d;
    const int64_t M = (p.T > (int64_t)blockIdx.x) ? (p.T - 1 - blockIdx.x) / G + 1 : 0;
    const int tile = sh.tile;
    const int ntile = sh.ntile;
    const int stages = sh.stages;
    const size_t row_bytes = (size_t)tile * sizeof(S);

    if (warp == 0) {
        // ---------------- producer ----------------
        if (lane != 0) return;
        const S *H = static_cast<const S *>(p.H);
        const S *Y = static_cast<const S *>(p.y);
        int64_t q = 0;
        bool ok = true;
        for (int64_t m = 0; m < M && ok; ++m) {
            const int64_t t = blockIdx.x + m * G;
            for (int j = 0; j < ntile; ++j, ++q) {
                const int slot = (int)(q % stages);
                const uint32_t ph = (uint32_t)((q / stages) & 1);
                if (q >= stages &&
                    !mbar_wait_bounded(&empty[slot], ph ^ 1u, abort_flag, fault, FAULT_WAIT_EMPTY)) {
                    ok = false;
                    break;
                }
                const int64_t k0 = (int64_t)j * tile;
                const int64_t w = (d - k0) < tile ? (d - k0) : tile;
                const uint32_t rb = (uint32_t)(w * (int64_t)sizeof(S));
                unsigned char *st = ring + (size_t)slot * sh.stage_bytes;
                mbar_arrive_expect_tx(&full[slot], rb * ROWS);
#pragma unroll
                for (int i = 0; i < N; ++i)
                    bulk_load(st + i * row_bytes, H + (t * N + i) * d + k0, rb, &full[slot]);
                if constexpr (WRITE) bulk_load(st + N * row_bytes, Y + t * d + k0, rb, &full[slot]);
            }
        }
        // every issued copy lands before the CTA may exit (normally already done)
        for (int64_t qq = (q > stages ? q - stages : 0); qq < q; ++qq)
            mbar_wait_drain(&full[qq % stages], (uint32_t)((qq / stages) & 1), fault);
        return;
    }

    if (warp == 1) {
        // ---------------- per-token parameters ----------------
        constexpr int GL = Group<N>::GL, EPL = Group<N>::EPL, TPW = Group<N>::TPW;
        const int q = lane & (GL - 1);
        for (int64_t m0 = 0; m0 < M; m0 += TPW) {
            const int64_t m = m0 + lane / GL;
            const bool live = m < M;
            const int64_t t = blockIdx.x + m * G;
            const int ps = (int)(m % kParamSlots);
            bool w = true;
            if (live && m >= kParamSlots)
                w = mbar_wait_bounded(&pempty[ps], (uint32_t)(((m / kParamSlots) & 1) ^ 1),
                                      abort_flag, fault, FAULT_WAIT_PARAM);
            if (!__all_sync(0xffffffffu, w)) break;
            float *P = params + ps * PSTRIDE;
            if constexpr (WRITE) {
                float mv[EPL];
#pragma unroll
                for (int r = 0; r < EPL; ++r) {
                    const int e = q + GL * r;
                    mv[r] = (live && e < NN) ? p.A[t * p.A_s + e] : 0.0f;
                }
                if (p.mix_logits) group_sinkhorn<N>(mv, lane, p.K);
                if (live) {
#pragma unroll
                    for (int r = 0; r < EPL; ++r) {
                        const int e = q + GL * r;
                        if (e < NN) P[e] = mv[r];
                    }
                    if (q < N) P[NN + q] = p.b[t * p.b_s + q];
                }
            }
            if constexpr (READ) {
                float l = (live && q < N) ? p.a[t * p.a_s + q] : 0.0f;
                if (p.read_logits) l = group_softmax<N>(l, lane);
                if (live && q < N) P[NN + N + q] = l;
            }
            __syncwarp();
            if (live && q == 0) mbar_arrive(&pfull[ps]);
        }
        return;
    }

    // ---------------- consumers ----------------
    const int cw = warp - 2;
    const int g = cw / GW;
    const int gw = cw - g * GW;
    const int gt = gw * 32 + lane;
    S *Ho = static_cast<S *>(p.Hout);
    S *X = static_cast<S *>(p.x);
    uint32_t ired = 0;  // tokens reduced by this group so far

    for (int64_t m = g; m < M; m += kPipeGroups) {
        const int64_t t = blockIdx.x + m * G;
        const int ps = (int)(m % kParamSlots);
        {
            const bool w = mbar_wait_bounded(&pfull[ps], (uint32_t)((m / kParamSlots) & 1),
                                             abort_flag, fault, FAULT_WAIT_PARAM);
            if (!__all_sync(0xffffffffu, w)) break;
        }
        const float *P = params + ps * PSTRIDE;
        float Ar[N <= 4 ? NN : 1];
        if constexpr (WRITE && N <= 4) {
#pragma unroll
            for (int e = 0; e < NN; ++e) Ar[e] = P[e];
        }
        float bv[N], av[N];
#pragma unroll
        for (int i = 0; i < N; ++i) {
            bv[i] = WRITE ? P[NN + i] : 0.0f;
            av[i] = READ ? P[NN + N + i] : 0.0f;
        }
        auto A_at = [&](int i, int j) -> float {
            if constexpr (N <= 4) return Ar[i * N + j];
            else return P[i * N + j];
        };

        bool ok = true;
        float hs[READ ? HT : 1][V];
        double ss = 0.0;
        int64_t q = m * ntile;

        auto do_tile = [&](int j) {
            const int slot = (int)(q % stages);
            const uint32_t ph = (uint32_t)((q / stages) & 1);
            ++q;
            const bool w = mbar_wait_bounded(&full[slot], ph, abort_flag, fault, FAULT_WAIT_FULL);
            if (!__all_sync(0xffffffffu, w)) {
                ok = false;
                return;
            }
            const unsigned char *st = ring + (size_t)slot * sh.stage_bytes + (size_t)gt * 16;
            const int64_t k = (int64_t)j * tile + (int64_t)gt * V;
            const bool active = k < d;
            float h[N][V], yv[V];
            if (active) {
#pragma unroll
                for (int i = 0; i < N; ++i) SmemVec<S>::load(st + i * row_bytes, h[i]);
                if constexpr (WRITE) SmemVec<S>::load(st + N * row_bytes, yv);
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(&empty[slot]);  // stage data is in registers
            if (!active) return;
            if constexpr (WRITE) {
                S *Hot = Ho + t * N * d + k;
                float hr[V];
#pragma unroll
                for (int e = 0; e < V; ++e) hr[e] = -0.0f;
#pragma unroll
                for (int jj = 0; jj < N; ++jj) {
                    float acc[V], stored[V];
#pragma unroll
                    for (int e = 0; e < V; ++e) acc[e] = -0.0f;
#pragma unroll
                    for (int i = 0; i < N; ++i) {
                        const float aij = A_at(i, jj);
#pragma unroll
                        for (int e = 0; e < V; ++e) acc[e] = __fmaf_rn(aij, h[i][e], acc[e]);
                    }
#pragma unroll
                    for (int e = 0; e < V; ++e) acc[e] = __fmaf_rn(bv[jj], yv[e], acc[e]);
                    store_vec_cs(Hot + jj * d, acc, stored);
                    if constexpr (READ) {
#pragma unroll
                        for (int e = 0; e < V; ++e) hr[e] = __fmaf_rn(av[jj], stored[e], hr[e]);
                    }
                }
                if constexpr (READ) {
#pragma unroll
                    for (int e = 0; e < V; ++e) hs[j][e] = hr[e];
                }
            } else {
#pragma unroll
                for (int e = 0; e < V; ++e) hs[j][e] = -0.0f;
#pragma unroll
                for (int i = 0; i < N; ++i) {
#pragma unroll
                    for (int e = 0; e < V; ++e) hs[j][e] = __fmaf_rn(av[i], h[i][e], hs[j][e]);
                }
            }
            if constexpr (READ) {
#pragma unroll
                for (int e = 0; e < V; ++e) {
                    const double hv = (double)hs[j][e];
                    ss = __fma_rn(hv, hv, ss);
                }
            }
        };

        if constexpr (READ) {
#pragma unroll
            for (int j = 0; j < HT; ++j) {
                if (j < ntile && ok) do_tile(j);
            }
        } else {
            for (int j = 0; j < ntile && ok; ++j) do_tile(j);
        }
        if (!ok) break;
        __syncwarp();
        if (lane == 0) mbar_arrive(&pempty[ps]);  // parameters no longer read

        if constexpr (READ) {
#pragma unroll
            for (int off = 16; off > 0; off >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, off);
            double *part = sred + (g * 2 + (ired & 1)) * GW;
            if (lane == 0) {
                part[gw] = ss;
                mbar_arrive(&redbar[g]);
            }
            const bool w = mbar_wait_bounded(&redbar[g], ired & 1, abort_flag, fault, FAULT_WAIT_REDUCE);
            if (!__all_sync(0xffffffffu, w)) break;
            ++ired;
            double tot = 0.0;
#pragma unroll
            for (int i = 0; i < GW; ++i) tot += part[i];
            const float r = __double2float_rn(1.0 / sqrt(tot / (double)d + (double)p.eps));
            S *Xt = X + t * d;
#pragma unroll
            for (int j = 0; j < HT; ++j) {
                const int64_t k = (int64_t)j * tile + (int64_t)gt * V;
                if (j < ntile && k < d) {
                    float gv[V], xv[V];
                    load_gain<V>(p.g, k, gv);
#pragma unroll
                    for (int e = 0; e < V; ++e) xv[e] = __fmul_rn(__fmul_rn(hs[j][e], r), gv[e]);
                    store_vec_cs(Xt + k, xv);
                }
            }
        }
    }
}

}  // namespace hc
