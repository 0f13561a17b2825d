// hc_pipe_kernels.cuh -- warp-specialised, TMA-fed kernels of the HC step.
//
// One persistent CTA per SM (tokens blockIdx.x, blockIdx.x + G, ...) with
// threads in three roles:
//   warp 0      producer: one lane streams each token's n stream rows (and y)
//               tile by tile into shared-memory stages with plain bulk copies
//               (cp.async.bulk, this GPU's own memory, no multicast),
//               completing on the stage's "full" mbarrier;
//   warp 1      parameters: lane groups compute the per-token Sinkhorn
//               projection / read softmax ahead of use into parameter slots;
//   warps 2..   consumer groups (kPipeGroups x kPipeGroupWarps warps); group
//               r owns tokens r, r + kPipeGroups, ... of the CTA, reads the
//               stages, writes H' with coalesced 128-bit stores, keeps h in an
//               fp32 shared-memory row, reduces the fp64 sum of squares across
//               its warps, then stores x.
// Every consumer group has its own ring of stages and its own parameter
// slots, so each mbarrier has exactly one consumer taking its phases in
// order (a parity wait is never more than one phase ahead). The producer
// serves the rings round-robin with non-blocking tests, so a slow group never
// holds back the others. HBM keeps tens of kilobytes per SM in flight while
// the consumers compute, reduce and store.
//
// Every wait is bounded (hc_sync.cuh): on time-out the CTA records a fault
// code, stops issuing, drains the copies it issued and exits.
#pragma once

#include "hc_device.cuh"
#include "hc_sync.cuh"

namespace hc {

// Consumer geometry (build-time constants; the defaults were chosen by
// measurement on B200 at n = 4, d = 7168, bf16).
#ifndef HC_PIPE_GROUPS
#define HC_PIPE_GROUPS 2
#endif
#ifndef HC_PIPE_GROUP_WARPS
#define HC_PIPE_GROUP_WARPS 7
#endif
constexpr int kPipeGroups = HC_PIPE_GROUPS;
constexpr int kPipeGroupWarps = HC_PIPE_GROUP_WARPS;
constexpr int kPipeGroupThreads = kPipeGroupWarps * 32;
constexpr int kPipeThreads = 64 + kPipeGroups * kPipeGroupThreads;
constexpr int kParamSlotsPerGroup = 8;
constexpr int kParamSlots = kParamSlotsPerGroup * kPipeGroups;
constexpr int kMaxStages = 32;
constexpr int kSmemLimit = 232448;  // 227 KB opt-in dynamic shared memory per CTA

struct PipeShape {
    int stages;       // stages in all (kPipeGroups rings of stages / kPipeGroups)
    int tile;         // elements of d per tile (= kPipeGroupThreads * V)
    int ntile;        // tiles per token
    int stage_bytes;  // bytes of one stage
};

// Bytes of everything in shared memory other than the ring: barriers,
// parameter slots, reduction partials, the abort flag and, for the
// normalising kinds, each group's fp32 row h[d] (d_h = d, else 0).
__host__ __device__ constexpr int64_t pipe_fixed_bytes(int n, int stages, int64_t d_h) {
    return (int64_t)stages * 16                        // full + empty barriers
           + kParamSlots * 16                          // param full + empty
           + (kPipeGroups + 1) / 2 * 16                // group reduction barriers
           + kParamSlots * (n * n + 2 * n) * 4         // parameter slots
           + kPipeGroups * 2 * kPipeGroupWarps * 8     // reduction partials
           + 16                                        // abort flag (padded)
           + (int64_t)kPipeGroups * ((d_h * 4 + 15) / 16 * 16);  // h rows
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

template <int N, typename S, int KIND>
__global__ void __launch_bounds__(kPipeThreads, 1)
hc_pipe_kernel(StepParams p, PipeShape sh, int *fault) {
    constexpr int V = StorageTraits<S>::V;
    constexpr int NN = N * N;
    constexpr bool WRITE = KIND != KIND_READ;
    constexpr bool READ = KIND != KIND_WRITE;
    constexpr int ROWS = WRITE ? N + 1 : N;
    constexpr int PSTRIDE = NN + 2 * N;  // A transposed (column j at j*N) | b | a
    constexpr int GW = kPipeGroupWarps;
    constexpr int NG = kPipeGroups;
    constexpr int PSG = kParamSlotsPerGroup;

    extern __shared__ __align__(128) unsigned char smem[];
    unsigned char *ring = smem;
    uint64_t *full = reinterpret_cast<uint64_t *>(smem + (size_t)sh.stages * sh.stage_bytes);
    uint64_t *empty = full + sh.stages;
    uint64_t *pfull = empty + sh.stages;
    uint64_t *pempty = pfull + kParamSlots;
    uint64_t *redbar = pempty + kParamSlots;
    float *params = reinterpret_cast<float *>(redbar + (NG + 1) / 2 * 2);
    double *sred = reinterpret_cast<double *>(params + kParamSlots * PSTRIDE);
    int *abort_word = reinterpret_cast<int *>(sred + NG * 2 * GW);
    volatile int *abort_flag = abort_word;
    float *hrow_base = reinterpret_cast<float *>(abort_word + 4);  // 16-byte aligned
    const int64_t d = p.d;
    const int64_t hrow_stride = READ ? (d + 3) / 4 * 4 : 0;  // floats per group row
    const int SG = sh.stages / NG;  // stages per group ring

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
        for (int g = 0; g < NG; ++g) mbar_init(&redbar[g], GW);
        *abort_flag = 0;
        fence_barrier_init();
    }
    __syncthreads();

    const int64_t G = gridDim.x;
    const int64_t M = (p.T > (int64_t)blockIdx.x) ? (p.T - 1 - blockIdx.x) / G + 1 : 0;
    const int tile = sh.tile;
    const int ntile = sh.ntile;
    const size_t row_bytes = (size_t)tile * sizeof(S);

    if (warp == 0) {
        // ---------------- producer ----------------
        if (lane != 0) return;
        const S *H = static_cast<const S *>(p.H);
        const S *Y = static_cast<const S *>(p.y);
        int64_t nq[NG], qend[NG];  // tiles issued / to issue, per group ring
#pragma unroll
        for (int r = 0; r < NG; ++r) {
            nq[r] = 0;
            qend[r] = (M > r ? (M - 1 - r) / NG + 1 : 0) * (int64_t)ntile;
        }
        uint64_t idle_since = 0;
        uint32_t idle_spins = 0;
        for (;;) {
            bool pending = false, progressed = false;
#pragma unroll
            for (int r = 0; r < NG; ++r) {
                const int64_t qr = nq[r];
                if (qr >= qend[r]) continue;
                pending = true;
                const int s = r * SG + (int)(qr % SG);
                if (qr >= SG && !mbar_test_wait(&empty[s], (uint32_t)(((qr / SG) & 1) ^ 1))) continue;
                const int64_t m = r + (qr / ntile) * NG;  // token ordinal within the CTA
                const int j = (int)(qr % ntile);
                const int64_t t = blockIdx.x + m * G;
                const int64_t k0 = (int64_t)j * tile;
                const int64_t w = (d - k0) < tile ? (d - k0) : tile;
                const uint32_t rb = (uint32_t)(w * (int64_t)sizeof(S));
                unsigned char *st = ring + (size_t)s * sh.stage_bytes;
                mbar_arrive_expect_tx(&full[s], rb * ROWS);
                const S *src = H + t * N * d + k0;
#pragma unroll
                for (int i = 0; i < N; ++i) bulk_load(st + i * row_bytes, src + i * d, rb, &full[s]);
                if constexpr (WRITE) bulk_load(st + N * row_bytes, Y + t * d + k0, rb, &full[s]);
                nq[r] = qr + 1;
                progressed = true;
            }
            if (!pending) break;
            if (progressed) {
                idle_since = 0;
                continue;
            }
            // every ring is full: back off; give up only after the time limit
            if (*abort_flag) break;
            if ((++idle_spins & 31u) == 0u) {
                const uint64_t now = global_timer_ns();
                if (idle_since == 0) {
                    idle_since = now;
                } else if (now - idle_since > kWaitLimitNs) {
                    *abort_flag = 1;
                    atomicOr(fault, FAULT_WAIT_EMPTY);
                    break;
                }
            }
            __nanosleep(32);
        }
        // every issued copy lands before the CTA may exit (normally already done)
#pragma unroll
        for (int r = 0; r < NG; ++r)
            for (int64_t qq = (nq[r] > SG ? nq[r] - SG : 0); qq < nq[r]; ++qq)
                mbar_wait_drain(&full[r * SG + (int)(qq % SG)], (uint32_t)((qq / SG) & 1), fault);
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
            const int64_t i = m / NG;  // token ordinal within its group
            const int ps = (int)(m % NG) * PSG + (int)(i % PSG);
            bool w = true;
            if (live && i >= PSG)
                w = mbar_wait_bounded(&pempty[ps], (uint32_t)(((i / PSG) & 1) ^ 1), abort_flag, fault,
                                      FAULT_WAIT_PARAM);
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
                        const int e = q + GL * r;  // A[i][j], i = e / N, j = e % N
                        if (e < NN) P[(e % N) * N + e / N] = mv[r];
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
    float *hrow = hrow_base + g * hrow_stride;  // this group's h[d] (fp32)
    uint64_t *gfull = full + g * SG;
    uint64_t *gempty = empty + g * SG;
    unsigned char *gring = ring + (size_t)g * SG * sh.stage_bytes;
    S *Ho = static_cast<S *>(p.Hout);
    S *X = static_cast<S *>(p.x);
    int64_t q = 0;  // tiles this group has consumed

    for (int64_t m = g, i = 0; m < M; m += NG, ++i) {
        const int64_t t = blockIdx.x + m * G;
        const int ps = g * PSG + (int)(i % PSG);
        {
            const bool w = mbar_wait_bounded(&pfull[ps], (uint32_t)((i / PSG) & 1), abort_flag, fault,
                                             FAULT_WAIT_PARAM);
            if (!__all_sync(0xffffffffu, w)) break;
        }
        const float *P = params + ps * PSTRIDE;
        float bv[N], av[N];
#pragma unroll
        for (int ii = 0; ii < N; ++ii) {
            bv[ii] = WRITE ? P[NN + ii] : 0.0f;
            av[ii] = READ ? P[NN + N + ii] : 0.0f;
        }

        bool ok = true;
        double ss = 0.0;
        S *Hot = Ho + t * N * d;
        for (int j = 0; j < ntile; ++j, ++q) {
            const int slot = (int)(q % SG);
            const uint32_t ph = (uint32_t)((q / SG) & 1);
            const bool w = mbar_wait_bounded(&gfull[slot], ph, abort_flag, fault, FAULT_WAIT_FULL);
            if (!__all_sync(0xffffffffu, w)) {
                ok = false;
                break;
            }
            const unsigned char *st = gring + (size_t)slot * sh.stage_bytes + (size_t)gt * 16;
            const int64_t k = (int64_t)j * tile + (int64_t)gt * V;
            const bool active = k < d;
            float h[N][V], yv[V];
            if (active) {
#pragma unroll
                for (int ii = 0; ii < N; ++ii) SmemVec<S>::load(st + ii * row_bytes, h[ii]);
                if constexpr (WRITE) SmemVec<S>::load(st + N * row_bytes, yv);
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(&gempty[slot]);  // stage data is in registers
            if (!active) continue;
            float hr[V];
            if constexpr (WRITE) {
#pragma unroll
                for (int jj = 0; jj < N; ++jj) {
                    // column jj of A: A[0][jj] .. A[N-1][jj]
                    float col[N];
#pragma unroll
                    for (int ii = 0; ii < N; ++ii) col[ii] = P[jj * N + ii];
                    float acc[V], stored[V];
#pragma unroll
                    for (int e = 0; e < V; ++e) acc[e] = __fmul_rn(col[0], h[0][e]);
#pragma unroll
                    for (int ii = 1; ii < N; ++ii) {
#pragma unroll
                        for (int e = 0; e < V; ++e) acc[e] = __fmaf_rn(col[ii], h[ii][e], acc[e]);
                    }
#pragma unroll
                    for (int e = 0; e < V; ++e) acc[e] = __fmaf_rn(bv[jj], yv[e], acc[e]);
                    store_vec_cs(Hot + jj * d + k, acc, stored);
                    if constexpr (READ) {
                        if (jj == 0) {
#pragma unroll
                            for (int e = 0; e < V; ++e) hr[e] = __fmul_rn(av[0], stored[e]);
                        } else {
#pragma unroll
                            for (int e = 0; e < V; ++e) hr[e] = __fmaf_rn(av[jj], stored[e], hr[e]);
                        }
                    }
                }
            } else {
#pragma unroll
                for (int e = 0; e < V; ++e) hr[e] = __fmul_rn(av[0], h[0][e]);
#pragma unroll
                for (int ii = 1; ii < N; ++ii) {
#pragma unroll
                    for (int e = 0; e < V; ++e) hr[e] = __fmaf_rn(av[ii], h[ii][e], hr[e]);
                }
            }
            if constexpr (READ) {
#pragma unroll
                for (int e = 0; e < V; ++e) {
                    const double hv = (double)hr[e];
                    ss = __fma_rn(hv, hv, ss);
                }
                // keep h for the normalisation (this thread reads it back itself)
#pragma unroll
                for (int e = 0; e < V; e += 4)
                    *reinterpret_cast<float4 *>(hrow + k + e) =
                        make_float4(hr[e], hr[e + 1], hr[e + 2], hr[e + 3]);
            }
        }
        if (!ok) break;
        __syncwarp();
        if (lane == 0) mbar_arrive(&pempty[ps]);  // parameters no longer read

        if constexpr (READ) {
#pragma unroll
            for (int off = 16; off > 0; off >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, off);
            double *part = sred + (g * 2 + (int)(i & 1)) * GW;
            if (lane == 0) {
                part[gw] = ss;
                mbar_arrive(&redbar[g]);
            }
            const bool w = mbar_wait_bounded(&redbar[g], (uint32_t)(i & 1), abort_flag, fault,
                                             FAULT_WAIT_REDUCE);
            if (!__all_sync(0xffffffffu, w)) break;
            double tot = 0.0;
#pragma unroll
            for (int ii = 0; ii < GW; ++ii) tot += part[ii];
            const float r = __double2float_rn(1.0 / sqrt(tot / (double)d + (double)p.eps));
            S *Xt = X + t * d;
            for (int j = 0; j < ntile; ++j) {
                const int64_t k = (int64_t)j * tile + (int64_t)gt * V;
                if (k < d) {
                    float gv[V], hv[V], xv[V];
                    load_gain<V>(p.g, k, gv);
#pragma unroll
                    for (int e = 0; e < V; e += 4) {
                        const float4 f = *reinterpret_cast<const float4 *>(hrow + k + e);
                        hv[e] = f.x; hv[e + 1] = f.y; hv[e + 2] = f.z; hv[e + 3] = f.w;
                    }
#pragma unroll
                    for (int e = 0; e < V; ++e) xv[e] = __fmul_rn(__fmul_rn(hv[e], r), gv[e]);
                    store_vec_cs(Xt + k, xv);
                }
            }
        }
    }
}

}  // namespace hc
