// hc_backward_pipe.cuh -- TMA-fed backward of the fused HC step (bf16, n <= 4).
//
// The same gradients as hc_step_bwd_kernel (hc_backward.cu), with the token's
// operands brought into shared memory by bulk copies instead of each thread's
// own loads, so the bytes in flight no longer depend on registers:
//
//   warp 0      producer: one lane bulk-copies (cp.async.bulk, this GPU's own
//               memory, no multicast) each token's H rows, y and dx, tile by
//               tile, into the token buffer (one region per tile of d), and
//               the gradient rows dH' into a ring of tiles;
//   warp 1      parameters: the forward's Sinkhorn projection and read softmax
//               per token (the fused step's parameter warp, one group);
//   warps 2..   consumers, one group taking the CTA's tokens in order. Pass 1
//               reads the token's tiles, recomputes H' (as stored) and h,
//               parks H' in shared memory and reduces sum h^2 and
//               sum g dx h (fp64) over the group; pass 2 reads the tiles again
//               (still in shared memory), forms dh, G, dH, dy and the
//               per-token sums, and releases each tile region to the
//               producer, which loads the next token's tile there while the
//               rest of pass 2 runs.
//
// One CTA per SM. Every wait is bounded (hc_sync.cuh): on time-out the CTA
// records a fault code, stops, drains the copies it issued and exits.
#pragma once

#include "hc_backward_common.cuh"
#include "hc_pipe_kernels.cuh"

namespace hc {

constexpr int kBwpConsumerWarps = 14;
constexpr int kBwpThreads = 64 + kBwpConsumerWarps * 32;
constexpr int kBwpVE = 4;  // bf16 elements per thread per row of a tile (8 bytes)
constexpr int kBwpTile = kBwpConsumerWarps * 32 * kBwpVE;
constexpr int kBwpGradStages = 3;
__host__ __device__ constexpr int bwp_param_slots(int n) {
    return ((2 * pipe_param_batch(n) > 8 ? 2 * pipe_param_batch(n) : 8) + 1) & ~1;
}

struct BwPipeShape {
    int ntile;        // tiles per token
    int gstages;      // dH' ring stages (0: no dH')
};

struct BwPipeParams {
    StepParams f;
    const void *dHout;
    const void *dx;
    void *dH;
    void *dy;
    float *gA, *gb, *ga;
    float *dg_part;  // [gridDim.x][d] or null
};

// Dynamic shared memory of the pipelined backward (bytes), laid out in this
// order: token buffer, dH' ring, parked H', gain partial, barriers,
// parameter slots, statistic and sum partials, abort flag, parameter scratch.
template <int N>
__host__ __device__ constexpr int64_t bwp_smem_bytes(int ntile, int gstages, bool want_dg) {
    constexpr int NN = N * N, NR = NN + 2 * N;
    const int64_t tb = (int64_t)kBwpTile * 2;  // bytes of one bf16 row of a tile
    return (int64_t)ntile * (N + 2) * tb                         // token buffer
           + (int64_t)gstages * N * tb                           // dH' ring
           + (int64_t)ntile * N * tb                             // parked H'
           + (want_dg ? (int64_t)ntile * kBwpTile * 4 : 0)       // gain partial
           + (int64_t)(2 * ntile + 2 * gstages + 2 * bwp_param_slots(N) + 4) * 8  // barriers
           + (int64_t)bwp_param_slots(N) * (NN + 2 * N) * 4      // parameter slots
           + 2 * kBwpConsumerWarps * 2 * 8                       // statistic partials (fp64)
           + ((2 * kBwpConsumerWarps * NR * 4 + 15) / 16 * 16)   // per-token sum partials
           + 16                                                  // abort flag
           + pipe_param_replicas(N) * kGroupScratch * 4;         // parameter warp scratch
}

template <int N>
__global__ void __launch_bounds__(kBwpThreads, 1)
hc_bwd_pipe_kernel(BwPipeParams bp, BwPipeShape sh, int *fault) {
    using S = __nv_bfloat16;
    using V = BwVec<S, kBwpVE>;
    constexpr int VE = kBwpVE;
    constexpr int NN = N * N, NR = NN + 2 * N;
    constexpr int CW = kBwpConsumerWarps;
    constexpr int PSG = bwp_param_slots(N);
    constexpr int PSTRIDE = NN + 2 * N;
    constexpr int TILE = kBwpTile;
    constexpr int64_t TB = (int64_t)TILE * 2;  // bytes of one row of a tile
    const StepParams &p = bp.f;
    const int ntile = sh.ntile;
    const int GS = sh.gstages;
    const bool want_dg = bp.dg_part != nullptr;
    const int64_t d = p.d;

    extern __shared__ __align__(128) unsigned char smem[];
    unsigned char *tok = smem;                                            // [ntile][N+2][TILE]
    unsigned char *gring = tok + (int64_t)ntile * (N + 2) * TB;           // [GS][N][TILE]
    unsigned char *hsb = gring + (int64_t)GS * N * TB;                    // [ntile][N][TILE]
    float *sdg = reinterpret_cast<float *>(hsb + (int64_t)ntile * N * TB);
    uint64_t *tfull = reinterpret_cast<uint64_t *>(reinterpret_cast<unsigned char *>(sdg) +
                                                   (want_dg ? (int64_t)ntile * TILE * 4 : 0));
    uint64_t *tempty = tfull + ntile;
    uint64_t *gfull = tempty + ntile;
    uint64_t *gempty = gfull + GS;
    uint64_t *pfull = gempty + GS;
    uint64_t *pempty = pfull + PSG;
    uint64_t *statbar = pempty + PSG;  // [2]
    uint64_t *sumbar = statbar + 2;    // [2]
    float *params = reinterpret_cast<float *>(sumbar + 2);
    double *statp = reinterpret_cast<double *>(params + PSG * PSTRIDE);  // [2][CW][2]
    float *sump = reinterpret_cast<float *>(statp + 2 * CW * 2);          // [2][CW][NR]
    int *abort_word = reinterpret_cast<int *>(
        reinterpret_cast<unsigned char *>(sump) + (2 * CW * NR * 4 + 15) / 16 * 16);
    volatile int *abort_flag = abort_word;
    float *pscratch = reinterpret_cast<float *>(abort_word + 4);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    if (threadIdx.x == 0) {
        for (int j = 0; j < ntile; ++j) {
            mbar_init(&tfull[j], 1);
            mbar_init(&tempty[j], CW);
        }
        for (int s = 0; s < GS; ++s) {
            mbar_init(&gfull[s], 1);
            mbar_init(&gempty[s], CW);
        }
        for (int s = 0; s < PSG; ++s) {
            mbar_init(&pfull[s], 1);
            mbar_init(&pempty[s], CW);
        }
        for (int s = 0; s < 2; ++s) {
            mbar_init(&statbar[s], CW);
            mbar_init(&sumbar[s], CW);
        }
        *abort_flag = 0;
        fence_barrier_init();
    }
    if (want_dg)
        for (int64_t k = threadIdx.x; k < (int64_t)ntile * TILE; k += blockDim.x) sdg[k] = 0.0f;
    __syncthreads();

    const int64_t G = gridDim.x;
    const int64_t M = (p.T > (int64_t)blockIdx.x) ? (p.T - 1 - blockIdx.x) / G + 1 : 0;

    if (warp == 0) {
        // ---------------- producer ----------------
        if (lane != 0) return;
        const S *H = static_cast<const S *>(p.H);
        const S *Y = static_cast<const S *>(p.y);
        const S *DX = static_cast<const S *>(bp.dx);
        const S *DHO = static_cast<const S *>(bp.dHout);
        const int64_t nq = M * ntile;  // tiles of each queue
        int64_t qt = 0, qg = 0;        // token tiles / dH' tiles issued
        uint64_t idle_since = 0;
        uint32_t backoff = 32;
        for (;;) {
            bool pending = false, progressed = false;
            if (qt < nq) {
                pending = true;
                const int64_t m = qt / ntile;
                const int j = (int)(qt - m * ntile);
                // region j is free once every consumer warp has finished token m-1 there
                if (m == 0 || mbar_test_wait(&tempty[j], (uint32_t)((m - 1) & 1))) {
                    const int64_t t = blockIdx.x + m * G;
                    const int64_t k0 = (int64_t)j * TILE;
                    const int64_t w = (d - k0) < TILE ? (d - k0) : TILE;
                    const uint32_t rb = (uint32_t)(w * 2);
                    unsigned char *rg = tok + (int64_t)j * (N + 2) * TB;
                    mbar_arrive_expect_tx(&tfull[j], rb * (N + 2));
#pragma unroll
                    for (int i = 0; i < N; ++i) bulk_load(rg + i * TB, H + (t * N + i) * d + k0, rb, &tfull[j]);
                    bulk_load(rg + N * TB, Y + t * d + k0, rb, &tfull[j]);
                    bulk_load(rg + (N + 1) * TB, DX + t * d + k0, rb, &tfull[j]);
                    ++qt;
                    progressed = true;
                }
            }
            if (GS > 0 && qg < nq) {
                pending = true;
                const int s = (int)(qg % GS);
                if (qg < GS || mbar_test_wait(&gempty[s], (uint32_t)(((qg / GS) & 1) ^ 1))) {
                    const int64_t m = qg / ntile;
                    const int j = (int)(qg - m * ntile);
                    const int64_t t = blockIdx.x + m * G;
                    const int64_t k0 = (int64_t)j * TILE;
                    const int64_t w = (d - k0) < TILE ? (d - k0) : TILE;
                    const uint32_t rb = (uint32_t)(w * 2);
                    unsigned char *rg = gring + (int64_t)s * N * TB;
                    mbar_arrive_expect_tx(&gfull[s], rb * N);
#pragma unroll
                    for (int i = 0; i < N; ++i) bulk_load(rg + i * TB, DHO + (t * N + i) * d + k0, rb, &gfull[s]);
                    ++qg;
                    progressed = true;
                }
            }
            if (!pending) break;
            if (progressed) {
                idle_since = 0;
                backoff = 32;
                continue;
            }
            if (*abort_flag) break;
            const uint64_t now = global_timer_ns();
            if (idle_since == 0) {
                idle_since = now;
            } else if (now - idle_since > kWaitLimitNs) {
                *abort_flag = 1;
                atomicOr(fault, FAULT_WAIT_EMPTY);
                break;
            }
            __nanosleep(backoff);
            if (backoff < 1024) backoff <<= 1;
        }
        // every issued copy lands before the CTA may exit (normally already done)
        for (int j = 0; j < ntile; ++j) {
            const int64_t fills = qt / ntile + (j < (int)(qt % ntile) ? 1 : 0);  // fills of region j
            if (fills > 0) mbar_wait_drain(&tfull[j], (uint32_t)((fills - 1) & 1), fault);
        }
        for (int64_t q = (qg > GS ? qg - GS : 0); q < qg; ++q)
            mbar_wait_drain(&gfull[(int)(q % GS)], (uint32_t)((q / GS) & 1), fault);
        return;
    }

    if (warp == 1) {
        pipe_param_warp<N, true, true, 1, PSG>(p, M, G, params, pfull, pempty, pscratch, abort_flag,
                                               fault, lane);
        return;
    }

    // ---------------- consumers ----------------
    const int cw = warp - 2;
    const int gt = cw * 32 + lane;  // this thread's slice of every tile
    S *DH = static_cast<S *>(bp.dH);
    S *DY = static_cast<S *>(bp.dy);
    int gslot = 0;
    uint32_t gph = 0;
    for (int64_t m = 0; m < M; ++m) {
        const int64_t t = blockIdx.x + m * G;
        const int ps = (int)(m % PSG);
        bool ok = mbar_wait_bounded(&pfull[ps], (uint32_t)((m / PSG) & 1), abort_flag, fault,
                                    FAULT_WAIT_PARAM);
        if (!__all_sync(0xffffffffu, ok)) break;
        // the slot holds A transposed (A[i][j] at j * N + i), then b, then a
        const float *P = params + ps * PSTRIDE;
        const float *bt = P + NN, *at = P + NN + N;

        // ---- pass 1: the token's statistics ----
        double ss = 0.0, sg = 0.0;
        for (int j = 0; j < ntile; ++j) {
            ok = mbar_wait_bounded(&tfull[j], (uint32_t)(m & 1), abort_flag, fault, FAULT_WAIT_FULL);
            if (!__all_sync(0xffffffffu, ok)) break;
            const int64_t k = (int64_t)j * TILE + (int64_t)gt * VE;
            if (k < d) {
                const unsigned char *rg = tok + (int64_t)j * (N + 2) * TB + (int64_t)gt * VE * 2;
                float hv[N][VE], yv[VE], hs[N][VE], h[VE], dxv[VE], gv[VE];
#pragma unroll
                for (int i = 0; i < N; ++i) V::load_smem(reinterpret_cast<const S *>(rg + i * TB), hv[i]);
                V::load_smem(reinterpret_cast<const S *>(rg + N * TB), yv);
                V::load_smem(reinterpret_cast<const S *>(rg + (N + 1) * TB), dxv);
                // H' as the forward stores it, and h (paired FMA chains)
#pragma unroll
                for (int e = 0; e < VE; ++e) h[e] = -0.0f;
#pragma unroll
                for (int jj = 0; jj < N; ++jj) {
#pragma unroll
                    for (int e = 0; e < VE; e += 2) {
                        float2 acc = make_float2(-0.0f, -0.0f);
#pragma unroll
                        for (int i = 0; i < N; ++i)
                            acc = ffma2_rn(make_float2(P[jj * N + i], P[jj * N + i]),
                                           make_float2(hv[i][e], hv[i][e + 1]), acc);
                        acc = ffma2_rn(make_float2(bt[jj], bt[jj]), make_float2(yv[e], yv[e + 1]), acc);
                        hs[jj][e] = acc.x;
                        hs[jj][e + 1] = acc.y;
                    }
                    V::round(hs[jj]);
#pragma unroll
                    for (int e = 0; e < VE; e += 2) {
                        const float2 hh = ffma2_rn(make_float2(at[jj], at[jj]),
                                                   make_float2(hs[jj][e], hs[jj][e + 1]),
                                                   make_float2(h[e], h[e + 1]));
                        h[e] = hh.x;
                        h[e + 1] = hh.y;
                    }
                    V::store_smem(reinterpret_cast<S *>(hsb + ((int64_t)j * N + jj) * TB +
                                                        (int64_t)gt * VE * 2),
                                  hs[jj]);
                }
                bw_load_gain<VE>(p.g, k, gv);
#pragma unroll
                for (int e = 0; e < VE; ++e) {
                    const double he = (double)h[e];
                    ss = __fma_rn(he, he, ss);
                    sg = __fma_rn((double)gv[e] * (double)dxv[e], he, sg);
                }
            }
        }
        if (!ok) break;
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) {
            ss += __shfl_xor_sync(0xffffffffu, ss, off);
            sg += __shfl_xor_sync(0xffffffffu, sg, off);
        }
        const int par = (int)(m & 1);
        if (lane == 0) {
            statp[(par * CW + cw) * 2] = ss;
            statp[(par * CW + cw) * 2 + 1] = sg;
            mbar_arrive(&statbar[par]);
        }
        ok = mbar_wait_bounded(&statbar[par], (uint32_t)((m >> 1) & 1), abort_flag, fault,
                               FAULT_WAIT_REDUCE);
        if (!__all_sync(0xffffffffu, ok)) break;
        double tss = 0.0, tsg = 0.0;
#pragma unroll
        for (int w = 0; w < CW; ++w) {
            tss += statp[(par * CW + w) * 2];
            tsg += statp[(par * CW + w) * 2 + 1];
        }
        const float r = __double2float_rn(1.0 / sqrt(tss / (double)d + (double)p.eps));
        const double rdd = (double)r;
        const float coef = (float)(rdd * rdd * rdd * tsg / (double)d);

        // ---- pass 2: gradients (the tiles are still in shared memory) ----
        // Per-thread partial sums. dA pairs streams (i, i+1) in one paired FMA
        // per element, db and da pair elements; every sum still takes its
        // terms in element order, as the register kernel's scalar chains do.
        constexpr int NP = (N + 1) / 2;  // stream pairs (the last half used for odd N)
        constexpr int VP = VE / 2;       // element pairs per slice
        float2 pA2[NP * N], pb2[N], pa2[N];
#pragma unroll
        for (int v = 0; v < NP * N; ++v) pA2[v] = make_float2(0.0f, 0.0f);
#pragma unroll
        for (int j = 0; j < N; ++j) {
            pb2[j] = make_float2(0.0f, 0.0f);
            pa2[j] = make_float2(0.0f, 0.0f);
        }
        const float2 r2 = make_float2(r, r), nc2 = make_float2(-coef, -coef);
        for (int j = 0; j < ntile; ++j) {
            const int cs = gslot;
            if (GS > 0) {
                ok = mbar_wait_bounded(&gfull[cs], gph, abort_flag, fault, FAULT_WAIT_FULL);
                if (!__all_sync(0xffffffffu, ok)) break;
                if (++gslot == GS) {
                    gslot = 0;
                    gph ^= 1u;
                }
            }
            const int64_t k = (int64_t)j * TILE + (int64_t)gt * VE;
            if (k < d) {
                const unsigned char *rg = tok + (int64_t)j * (N + 2) * TB + (int64_t)gt * VE * 2;
                const unsigned char *hg = hsb + (int64_t)j * N * TB + (int64_t)gt * VE * 2;
                float hv[N][VE], yv[VE], hsk[N][VE], dxv[VE], gv[VE];
#pragma unroll
                for (int i = 0; i < N; ++i) V::load_smem(reinterpret_cast<const S *>(rg + i * TB), hv[i]);
                V::load_smem(reinterpret_cast<const S *>(rg + N * TB), yv);
                V::load_smem(reinterpret_cast<const S *>(rg + (N + 1) * TB), dxv);
#pragma unroll
                for (int jj = 0; jj < N; ++jj) V::load_smem(reinterpret_cast<const S *>(hg + jj * TB), hsk[jj]);
                bw_load_gain<VE>(p.g, k, gv);
                // h from the parked H', then dh = r g dx - coef h (paired, element-wise
                // the scalar operations)
                float2 h2[VP], dh2[VP];
#pragma unroll
                for (int q = 0; q < VP; ++q) h2[q] = make_float2(-0.0f, -0.0f);
#pragma unroll
                for (int jj = 0; jj < N; ++jj)
#pragma unroll
                    for (int q = 0; q < VP; ++q)
                        h2[q] = ffma2_rn(make_float2(at[jj], at[jj]),
                                         make_float2(hsk[jj][2 * q], hsk[jj][2 * q + 1]), h2[q]);
#pragma unroll
                for (int q = 0; q < VP; ++q) {
                    const float2 dx2 = make_float2(dxv[2 * q], dxv[2 * q + 1]);
                    dh2[q] = ffma2_rn(nc2, h2[q],
                                      fmul2_rn(fmul2_rn(r2, make_float2(gv[2 * q], gv[2 * q + 1])), dx2));
                    if (want_dg) {
                        float2 *dgk = reinterpret_cast<float2 *>(sdg + (int64_t)j * TILE + (int64_t)gt * VE) + q;
                        *dgk = ffma2_rn(fmul2_rn(dx2, h2[q]), r2, *dgk);
                    }
                }
                float2 dH2[N][VP], dy2[VP];
#pragma unroll
                for (int q = 0; q < VP; ++q) dy2[q] = make_float2(0.0f, 0.0f);
#pragma unroll
                for (int i = 0; i < N; ++i)
#pragma unroll
                    for (int q = 0; q < VP; ++q) dH2[i][q] = make_float2(0.0f, 0.0f);
#pragma unroll
                for (int jj = 0; jj < N; ++jj) {
                    float Gj[VE];
                    if (GS > 0) {
                        V::load_smem(reinterpret_cast<const S *>(gring + ((int64_t)cs * N + jj) * TB +
                                                                 (int64_t)gt * VE * 2),
                                     Gj);
                    } else {
#pragma unroll
                        for (int e = 0; e < VE; ++e) Gj[e] = 0.0f;
                    }
                    const float2 aj2 = make_float2(at[jj], at[jj]), bj2 = make_float2(bt[jj], bt[jj]);
#pragma unroll
                    for (int q = 0; q < VP; ++q) {
                        const float2 G2 = ffma2_rn(aj2, dh2[q], make_float2(Gj[2 * q], Gj[2 * q + 1]));
                        pa2[jj] = ffma2_rn(dh2[q], make_float2(hsk[jj][2 * q], hsk[jj][2 * q + 1]), pa2[jj]);
                        pb2[jj] = ffma2_rn(make_float2(yv[2 * q], yv[2 * q + 1]), G2, pb2[jj]);
                        dy2[q] = ffma2_rn(bj2, G2, dy2[q]);
#pragma unroll
                        for (int i = 0; i < N; ++i) {
                            const float aij = P[jj * N + i];
                            dH2[i][q] = ffma2_rn(make_float2(aij, aij), G2, dH2[i][q]);
                        }
#pragma unroll
                        for (int ip = 0; ip < NP; ++ip) {
                            const int i0 = 2 * ip, i1 = 2 * ip + 1;
                            float2 &acc = pA2[ip * N + jj];
                            acc = ffma2_rn(make_float2(hv[i0][2 * q], i1 < N ? hv[i1 < N ? i1 : i0][2 * q] : 0.0f),
                                           make_float2(G2.x, G2.x), acc);
                            acc = ffma2_rn(make_float2(hv[i0][2 * q + 1],
                                                       i1 < N ? hv[i1 < N ? i1 : i0][2 * q + 1] : 0.0f),
                                           make_float2(G2.y, G2.y), acc);
                        }
                    }
                }
#pragma unroll
                for (int i = 0; i < N; ++i) {
                    float o[VE];
#pragma unroll
                    for (int q = 0; q < VP; ++q) {
                        o[2 * q] = dH2[i][q].x;
                        o[2 * q + 1] = dH2[i][q].y;
                    }
                    V::store(DH + (t * N + i) * d + k, o);
                }
                float o[VE];
#pragma unroll
                for (int q = 0; q < VP; ++q) {
                    o[2 * q] = dy2[q].x;
                    o[2 * q + 1] = dy2[q].y;
                }
                V::store(DY + t * d + k, o);
            }
            __syncwarp();
            if (lane == 0) {
                mbar_arrive(&tempty[j]);  // the producer may load the next token's tile here
                if (GS > 0) mbar_arrive(&gempty[cs]);
            }
        }
        if (!ok) break;
        __syncwarp();
        if (lane == 0) mbar_arrive(&pempty[ps]);  // parameters no longer read
        // per-token sums: warp trees (fp32), then the warps in order (fp64)
#pragma unroll
        for (int v = 0; v < NR; ++v) {
            float val;
            if (v < NN) {
                const int i = v / N, jj = v - (v / N) * N;  // dA[i][jj]
                val = (i & 1) ? pA2[(i >> 1) * N + jj].y : pA2[(i >> 1) * N + jj].x;
            } else {
                const float2 pv = v < NN + N ? pb2[v - NN] : pa2[v - NN - N];
                val = __fadd_rn(pv.x, pv.y);
            }
#pragma unroll
            for (int off = 16; off > 0; off >>= 1) val += __shfl_xor_sync(0xffffffffu, val, off);
            if (lane == 0) sump[(par * CW + cw) * NR + v] = val;
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&sumbar[par]);
        if (cw == 0) {
            ok = mbar_wait_bounded(&sumbar[par], (uint32_t)((m >> 1) & 1), abort_flag, fault,
                                   FAULT_WAIT_REDUCE);
            if (!__all_sync(0xffffffffu, ok)) break;
            if (lane < NR) {
                double acc = 0.0;
#pragma unroll
                for (int w = 0; w < CW; ++w) acc += (double)sump[(par * CW + w) * NR + lane];
                const float out = (float)acc;
                if (lane < NN) bp.gA[t * NN + lane] = out;
                else if (lane < NN + N) bp.gb[t * N + (lane - NN)] = out;
                else bp.ga[t * N + (lane - NN - N)] = out;
            }
        }
    }
    if (want_dg) {
        // every consumer thread wrote only its own slices: each writes them out
        for (int j = 0; j < ntile; ++j) {
            const int64_t k = (int64_t)j * TILE + (int64_t)gt * VE;
            if (k < d) {
#pragma unroll
                for (int e = 0; e < VE; ++e)
                    bp.dg_part[(int64_t)blockIdx.x * d + k + e] = sdg[(int64_t)j * TILE + (int64_t)gt * VE + e];
            }
        }
    }
}

}  // namespace hc
