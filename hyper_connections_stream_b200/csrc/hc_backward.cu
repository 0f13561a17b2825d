// hc_backward.cu -- backward pass of the fused HC step (training).
//
// Gradients of  H'_j = sum_i A[i][j] H_i + b_j y,  h = sum_j a_j H'_j,
// x = h r g,  r = (sum h^2 / d + eps)^(-1/2)  (the forward of
// hc_write_then_read; the glossary entry "Hyper-connections (mHC)": learned
// mixing before and after each block, Sinkhorn-projected in mHC), straight
// through the storage rounding:
//   dh = r g dx - (r^3 / d) h sum(g dx h)       G_j = dH'_j + a_j dh
//   dH_i = sum_j A[i][j] G_j    dy = sum_j b_j G_j    dg = sum_t dx h r
//   dA[i][j] = sum_k H_i G_j    db_j = sum_k y G_j    da_j = sum_k dh H'_j
// then per token through the read softmax and the Sinkhorn projection.
//
// Kernels:
//   hc_step_bwd_kernel   one CTA per token at a time (grid-stride), threads own
//                        column slices, their global rows staged ahead through
//                        a per-thread cp.async ring. Phase 1 recomputes H' (as
//                        stored) and h, reduces sum h^2 and sum g dx h (fp64)
//                        and the two da sums, and parks h in shared memory;
//                        phase 2 re-reads H, y, dx (L2-resident by then),
//                        reads dH', forms dh, G, dH, dy and the dA / db sums
//                        (fp32 per thread, fp64 across warps); the gain
//                        gradient accumulates in the CTA's workspace row.
//   hc_param_bwd_kernel  lane group per token: the softmax backward, and the
//                        Sinkhorn backward with the 2K+1 iterates kept in
//                        shared memory; in place on dA / da.
//   hc_dg_reduce_kernel  sums the per-CTA gain partials in a fixed order.
#include <atomic>

#include "hc_launch.h"
#include "hc_backward_common.cuh"
#include "hc_backward_pipe.cuh"

namespace hc {

namespace {

constexpr int kBwTB = 32;       // parameter slots per batch
constexpr int kBwThreads = 256;  // largest CTA of the step kernel

#define HC_BW_TRY(expr)                 \
    do {                                \
        hc_status _st = (expr);         \
        if (_st != HC_OK) return _st;   \
    } while (0)

// One CTA per token at a time (grid-stride over tokens), threads own VE-wide
// column slices; two CTAs per SM (128 registers a thread) up to n = 5, the
// n*n per-thread sums of larger n need the full register file.
//
// Phase 1 recomputes H' (as stored) and h, reduces sum h^2 and sum g dx h
// (fp64), and forms the read-weight gradient while H' is live:
//   da_j = sum_k dh H'_j = r sum_k (g dx) H'_j - (r^3/d)(sum g dx h) sum_k h H'_j
// (both sums finished once r and the coefficient are known). Phase 2 then
// needs h but not H': PARK keeps h (fp32, d * 4 bytes) in shared memory from
// phase 1 (each thread reads back only the slots it wrote), otherwise phase 2
// rebuilds h from H and y. Phase 2 re-reads H, y and dx (from L2), reads dH',
// and forms dh, G, dH, dy and the dA / db sums (fp32 per thread, dA paired
// over stream pairs; one halving exchange per warp, fp64 across warps). The
// gain gradient accumulates in this CTA's workspace row.
//
// RING > 0: each thread stages the global rows of its next RING - 1 slices
// (H, y, dx and, in phase 2, dH') in its own shared-memory slots with
// cp.async, in the order the loops consume them (phase 1 then phase 2 of
// each token, tokens in order), so every thread keeps loads in flight while
// it computes instead of waiting for each slice's loads.
template <int N, typename S, int VE, bool PARK, int RING>
__global__ void __launch_bounds__(kBwThreads, (N <= 5 ? 2 : 1))
hc_step_bwd_kernel(BwKernelParams bp) {
    const StepParams &p = bp.f;
    constexpr int NN = N * N;
    constexpr int NS = NN + N;  // phase-2 sums: dA, db
    constexpr int NP = (N + 1) / 2;
    static_assert(RING == 0 || (RING >= 2 && PARK), "a ring needs two stages and the parked h");
    using V = BwVec<S, VE>;
    __shared__ float sA[kBwTB * NN], sb[kBwTB * N], sa[kBwTB * N];
    __shared__ double sred[2][kBwThreads / 32];
    __shared__ float pred1[kBwThreads / 32][2 * N];
    __shared__ float pred[kBwThreads / 32][NS];
    __shared__ float swork[kBwThreads / 32 * kGroupScratch];
    extern __shared__ __align__(16) unsigned char bw_dyn[];

    const int tid = threadIdx.x;
    const int NT = blockDim.x;
    const int nwarps = NT >> 5;
    const int lane = tid & 31, warp = tid >> 5;
    const int64_t d = p.d;
    const int64_t nvec = d / VE;
    const int64_t G = gridDim.x;
    int TB = nwarps * Group<N>::TPW;
    TB = TB < kBwTB ? TB : kBwTB;

    const S *H = static_cast<const S *>(p.H);
    const S *Y = static_cast<const S *>(p.y);
    const S *DX = static_cast<const S *>(bp.dx);
    const S *DHO = static_cast<const S *>(bp.dHout);
    S *DH = static_cast<S *>(bp.dH);
    S *DY = static_cast<S *>(bp.dy);
    const bool want_dg = bp.dg_part != nullptr;
    // The gain partial accumulates in this CTA's workspace row (L2-resident:
    // grid x d x 4 bytes); each thread reads and writes only the slots of its
    // own slices, in program order.
    float *sdg = want_dg ? bp.dg_part + (int64_t)blockIdx.x * d : nullptr;
    if (want_dg)
        for (int64_t c = tid; c < nvec; c += NT) {
            const float z[VE] = {};
            bw_st_f32<VE>(sdg + c * VE, z);
        }
    float *shp = reinterpret_cast<float *>(bw_dyn);  // [d] parked h

    // Staging ring: [RING slots][2N + 2 rows: H, y, dx, dH'][NT threads]
    // chunks of VE elements, so a warp's copies of one row land contiguously.
    constexpr int RR = 2 * N + 2;
    constexpr int CB = VE * (int)sizeof(S);
    const int ROW = NT * CB;
    unsigned char *ring0 = bw_dyn + (PARK ? d * 4 : 0);
    auto slot = [&](int st, int row) -> unsigned char * {
        return ring0 + ((size_t)(st * RR + row) * NT + tid) * CB;
    };
    // next slice to stage: slice pc of phase pph of token blockIdx.x + pm G
    int64_t pm = 0, pc = tid;
    int pph = 0, ist = 0, cst = 0;
    auto stage_next = [&]() {
        if constexpr (RING > 0) {
            const int64_t tq = blockIdx.x + pm * G;
            if (pc < nvec && tq < p.T) {
                const int64_t k = pc * VE;
#pragma unroll
                for (int i = 0; i < N; ++i)
                    bw_cp_async<CB>(smem_addr(slot(ist, i)), H + (tq * N + i) * d + k);
                bw_cp_async<CB>(smem_addr(slot(ist, N)), Y + tq * d + k);
                bw_cp_async<CB>(smem_addr(slot(ist, N + 1)), DX + tq * d + k);
                if (pph == 1 && DHO) {
#pragma unroll
                    for (int j = 0; j < N; ++j)
                        bw_cp_async<CB>(smem_addr(slot(ist, N + 2 + j)), DHO + (tq * N + j) * d + k);
                }
            }
            bw_cp_commit();  // possibly empty: one group per slice keeps the count
            ist = ist + 1 == RING ? 0 : ist + 1;
            pc += NT;
            if (pc >= nvec) {
                pc = tid;
                if (pph == 0) {
                    pph = 1;
                } else {
                    pph = 0;
                    ++pm;
                }
            }
        }
    };
    // The slot of the next slice to compute, once its copies have landed;
    // then the slice RING - 1 ahead is staged into the slot read last.
    // (Measured: per-token row bases with constant slot offsets issue 18 %
    // fewer instructions but ran 10 % slower, as did staging before the wait.)
    auto take = [&]() -> const unsigned char * {
        bw_cp_wait<RING >= 2 ? RING - 2 : 0>();
        stage_next();
        const int st = cst;
        cst = cst + 1 == RING ? 0 : cst + 1;
        return slot(st, 0);
    };
    if constexpr (RING > 0) {
        for (int q = 0; q < RING - 1; ++q) stage_next();
    }

    for (int64_t m0 = 0;; m0 += TB) {
        const int64_t first = blockIdx.x + m0 * G;
        if (first >= p.T) break;
        __syncthreads();  // previous batch's parameters no longer read
        prepare_params<N, true, true>(p, first, G, TB, sA, sb, sa, swork);
        __syncthreads();
        for (int tt = 0; tt < TB; ++tt) {
            const int64_t t = first + (int64_t)tt * G;
            if (t >= p.T) break;  // uniform over the CTA
            const float *At = sA + tt * NN, *bt = sb + tt * N, *at = sa + tt * N;
            const S *Ht = H + t * N * d, *Yt = Y + t * d, *DXt = DX + t * d;

            // ---- phase 1: the token's statistics and the da sums ----
            double ss = 0.0, sg = 0.0;
            float2 s1[N], s2[N];
#pragma unroll
            for (int j = 0; j < N; ++j) {
                s1[j] = make_float2(0.0f, 0.0f);
                s2[j] = make_float2(0.0f, 0.0f);
            }
            for (int64_t c = tid; c < nvec; c += NT) {
                const int64_t k = c * VE;
                float hv[N][VE], yv[VE], hs[N][VE], h[VE], dxv[VE], gv[VE];
                if constexpr (RING > 0) {
                    const unsigned char *sp = take();
#pragma unroll
                    for (int i = 0; i < N; ++i) bw_ld_stage<S, VE>(sp + i * ROW, hv[i]);
                    bw_ld_stage<S, VE>(sp + N * ROW, yv);
                    bw_ld_stage<S, VE>(sp + (N + 1) * ROW, dxv);
                    bw_forward_from<N, S, VE>(hv, yv, At, bt, at, hs, h);
                } else {
                    bw_forward_slice<N, S, VE>(Ht, Yt, d, k, At, bt, at, hv, yv, hs, h);
                    V::load(DXt + k, dxv);
                }
                if constexpr (PARK) bw_st_f32<VE>(shp + k, h);
                bw_load_gain<VE>(p.g, k, gv);
#pragma unroll
                for (int e = 0; e < VE; e += 2) {
                    const float2 gdx = fmul2_rn(make_float2(gv[e], gv[e + 1]), make_float2(dxv[e], dxv[e + 1]));
                    const float2 h2 = make_float2(h[e], h[e + 1]);
#pragma unroll
                    for (int j = 0; j < N; ++j) {
                        const float2 hs2 = make_float2(hs[j][e], hs[j][e + 1]);
                        s1[j] = ffma2_rn(gdx, hs2, s1[j]);
                        s2[j] = ffma2_rn(h2, hs2, s2[j]);
                    }
                }
#pragma unroll
                for (int e = 0; e < VE; ++e) {
                    const double he = (double)h[e];
                    ss = __fma_rn(he, he, ss);
                    sg = __fma_rn((double)gv[e] * (double)dxv[e], he, sg);
                }
            }
#pragma unroll
            for (int off = 16; off > 0; off >>= 1) {
                ss += __shfl_xor_sync(0xffffffffu, ss, off);
                sg += __shfl_xor_sync(0xffffffffu, sg, off);
            }
            {
                float v1[2 * N];
#pragma unroll
                for (int j = 0; j < N; ++j) {
                    v1[j] = __fadd_rn(s1[j].x, s1[j].y);
                    v1[N + j] = __fadd_rn(s2[j].x, s2[j].y);
                }
                if constexpr (2 * N <= 32) {
                    bw_warp_sums_to<2 * N>(v1, pred1[warp], lane);
                } else {
#pragma unroll
                    for (int v = 0; v < 2 * N; ++v) {
                        float val = v1[v];
#pragma unroll
                        for (int off = 16; off > 0; off >>= 1) val += __shfl_xor_sync(0xffffffffu, val, off);
                        if (lane == 0) pred1[warp][v] = val;
                    }
                }
            }
            if (lane == 0) {
                sred[0][warp] = ss;
                sred[1][warp] = sg;
            }
            __syncthreads();
            double tss = 0.0, tsg = 0.0;
            for (int w = 0; w < nwarps; ++w) {
                tss += sred[0][w];
                tsg += sred[1][w];
            }
            const float r = __double2float_rn(1.0 / sqrt(tss / (double)d + (double)p.eps));
            const double rd = (double)r;
            const float coef = (float)(rd * rd * rd * tsg / (double)d);
            if (tid < N) {
                double S1 = 0.0, S2 = 0.0;
                for (int w = 0; w < nwarps; ++w) {
                    S1 += (double)pred1[w][tid];
                    S2 += (double)pred1[w][N + tid];
                }
                bp.ga[t * N + tid] = (float)(rd * S1 - (double)coef * S2);
            }

            // ---- phase 2: gradients (H, y, dx and dH' read; the first three from L2) ----
            float2 pA2[N][NP];
#pragma unroll
            for (int i = 0; i < N; ++i)
#pragma unroll
                for (int q = 0; q < NP; ++q) pA2[i][q] = make_float2(0.0f, 0.0f);
            float2 pb2[N];
#pragma unroll
            for (int j = 0; j < N; ++j) pb2[j] = make_float2(0.0f, 0.0f);
            const float2 r2 = make_float2(r, r), nc2 = make_float2(-coef, -coef);
            for (int64_t c = tid; c < nvec; c += NT) {
                const int64_t k = c * VE;
                float hv[N][VE], yv[VE], h[VE], dh[VE], dxv[VE];
                const unsigned char *sp = nullptr;
                if constexpr (RING > 0) {
                    sp = take();
#pragma unroll
                    for (int i = 0; i < N; ++i) bw_ld_stage<S, VE>(sp + i * ROW, hv[i]);
                    bw_ld_stage<S, VE>(sp + N * ROW, yv);
                    bw_ld_stage<S, VE>(sp + (N + 1) * ROW, dxv);
                } else {
#pragma unroll
                    for (int i = 0; i < N; ++i) V::load(Ht + i * d + k, hv[i]);
                    V::load(Yt + k, yv);
                    V::load(DXt + k, dxv);
                }
                if constexpr (PARK) {
                    bw_ld_f32<VE>(shp + k, h);
                } else {
#pragma unroll
                    for (int e = 0; e < VE; ++e) h[e] = -0.0f;
#pragma unroll
                    for (int j = 0; j < N; ++j) {
                        float hs[VE];
                        bw_stream_out<N, S, VE>(hv, yv, At, bt, j, hs);
#pragma unroll
                        for (int e = 0; e < VE; ++e) h[e] = __fmaf_rn(at[j], hs[e], h[e]);
                    }
                }
                {
                    float gv[VE];
                    bw_load_gain<VE>(p.g, k, gv);
                    float sd[VE];
                    if (want_dg) bw_ld_f32<VE>(sdg + k, sd);
#pragma unroll
                    for (int e = 0; e < VE; e += 2) {
                        const float2 dx2 = make_float2(dxv[e], dxv[e + 1]);
                        const float2 h2 = make_float2(h[e], h[e + 1]);
                        const float2 u = fmul2_rn(fmul2_rn(r2, make_float2(gv[e], gv[e + 1])), dx2);
                        const float2 dh2 = ffma2_rn(nc2, h2, u);
                        dh[e] = dh2.x;
                        dh[e + 1] = dh2.y;
                        if (want_dg) {
                            const float2 s = ffma2_rn(fmul2_rn(dx2, h2), r2, make_float2(sd[e], sd[e + 1]));
                            sd[e] = s.x;
                            sd[e + 1] = s.y;
                        }
                    }
                    if (want_dg) bw_st_f32<VE>(sdg + k, sd);
                }
                float dHacc[N][VE], dyacc[VE];
#pragma unroll
                for (int e = 0; e < VE; ++e) dyacc[e] = 0.0f;
#pragma unroll
                for (int i = 0; i < N; ++i)
#pragma unroll
                    for (int e = 0; e < VE; ++e) dHacc[i][e] = 0.0f;
#pragma unroll
                for (int jp = 0; jp < NP; ++jp) {
                    float Gq[2][VE];
#pragma unroll
                    for (int q = 0; q < 2; ++q) {
                        const int j = 2 * jp + q;
                        if (j >= N) break;
                        if (DHO) {
                            if constexpr (RING > 0) bw_ld_stage<S, VE>(sp + (N + 2 + j) * ROW, Gq[q]);
                            else V::load(DHO + (t * N + j) * d + k, Gq[q]);
                        } else {
#pragma unroll
                            for (int e = 0; e < VE; ++e) Gq[q][e] = 0.0f;
                        }
#pragma unroll
                        for (int e = 0; e < VE; e += 2) {
                            const float2 G2 = ffma2_rn(make_float2(at[j], at[j]), make_float2(dh[e], dh[e + 1]),
                                                       make_float2(Gq[q][e], Gq[q][e + 1]));
                            Gq[q][e] = G2.x;
                            Gq[q][e + 1] = G2.y;
                            pb2[j] = ffma2_rn(make_float2(yv[e], yv[e + 1]), G2, pb2[j]);
                            const float2 dy2 = ffma2_rn(make_float2(bt[j], bt[j]), G2,
                                                        make_float2(dyacc[e], dyacc[e + 1]));
                            dyacc[e] = dy2.x;
                            dyacc[e + 1] = dy2.y;
#pragma unroll
                            for (int i = 0; i < N; ++i) {
                                const float aij = At[i * N + j];
                                const float2 dH2 = ffma2_rn(make_float2(aij, aij), G2,
                                                            make_float2(dHacc[i][e], dHacc[i][e + 1]));
                                dHacc[i][e] = dH2.x;
                                dHacc[i][e + 1] = dH2.y;
                            }
                        }
                    }
                    // dA[i][2jp], dA[i][2jp+1]: one paired FMA per element, each
                    // half the scalar chain over the slice's elements in order
#pragma unroll
                    for (int e = 0; e < VE; ++e)
#pragma unroll
                        for (int i = 0; i < N; ++i) {
                            if (2 * jp + 1 < N)
                                pA2[i][jp] = ffma2_rn(make_float2(hv[i][e], hv[i][e]),
                                                      make_float2(Gq[0][e], Gq[1][e]), pA2[i][jp]);
                            else
                                pA2[i][jp].x = __fmaf_rn(hv[i][e], Gq[0][e], pA2[i][jp].x);
                        }
                }
#pragma unroll
                for (int i = 0; i < N; ++i) V::store(DH + (t * N + i) * d + k, dHacc[i]);
                V::store(DY + t * d + k, dyacc);
            }
            // per-token sums: warp sums (fp32), then the warps in order (fp64)
            {
                float v2[NS];
#pragma unroll
                for (int i = 0; i < N; ++i)
#pragma unroll
                    for (int j = 0; j < N; ++j) {
                        v2[i * N + j] = (j & 1) ? pA2[i][j >> 1].y : pA2[i][j >> 1].x;
                    }
#pragma unroll
                for (int j = 0; j < N; ++j) v2[NN + j] = __fadd_rn(pb2[j].x, pb2[j].y);
                if constexpr (NS <= 32) {
                    bw_warp_sums_to<NS>(v2, pred[warp], lane);
                } else {
#pragma unroll
                    for (int v = 0; v < NS; ++v) {
                        float val = v2[v];
#pragma unroll
                        for (int off = 16; off > 0; off >>= 1) val += __shfl_xor_sync(0xffffffffu, val, off);
                        if (lane == 0) pred[warp][v] = val;
                    }
                }
            }
            __syncthreads();
            if (tid < NS) {
                double acc = 0.0;
                for (int w = 0; w < nwarps; ++w) acc += (double)pred[w][tid];
                const float out = (float)acc;
                if (tid < NN) bp.gA[t * NN + tid] = out;
                else bp.gb[t * N + (tid - NN)] = out;
            }
        }
    }
    if constexpr (RING > 0) bw_cp_wait_all();
}

// Per token, in place: da <- softmax backward of da (read logits), dA <- the
// Sinkhorn backward of dA (mixing logits). Lane groups as in the forward's
// parameter preparation; the 2K+1 Sinkhorn iterates of every lane live in
// dynamic shared memory.
template <int N>
__global__ void __launch_bounds__(128)
hc_param_bwd_kernel(const float *L, int64_t L_s, const float *l, int64_t l_s, float *dA, float *da,
                    int64_t T, int K, int mix, int read) {
    constexpr int NN = N * N, GL = Group<N>::GL, EPL = Group<N>::EPL, TPW = Group<N>::TPW;
    extern __shared__ float hist[];  // [(2K+1)][blockDim.x][EPL]
    __shared__ float sw[4][2 * 64];
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int q = lane & (GL - 1);
    float *buf = sw[warp] + (lane / GL) * NN;       // values of the group's matrix
    float *buf2 = sw[warp] + 64 + (lane / GL) * NN;  // second exchange buffer
    const int64_t wg = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    const int64_t nw = ((int64_t)gridDim.x * blockDim.x) >> 5;
    int e[EPL], row[EPL], col[EPL];
    bool own[EPL];
#pragma unroll
    for (int r = 0; r < EPL; ++r) {
        e[r] = q + GL * r;
        own[r] = e[r] < NN;
        const int ec = own[r] ? e[r] : NN - 1;
        row[r] = ec / N;
        col[r] = ec - row[r] * N;
    }
    for (int64_t t0 = wg * TPW; t0 < T; t0 += nw * TPW) {
        const int64_t t = t0 + lane / GL;
        const bool live = t < T;
        if (mix) {
            float m[EPL], g[EPL];
#pragma unroll
            for (int r = 0; r < EPL; ++r) {
                m[r] = expf((live && own[r]) ? L[t * L_s + e[r]] : 0.0f);
                g[r] = (live && own[r]) ? dA[t * NN + e[r]] : 0.0f;
                hist[((int64_t)0 * blockDim.x + threadIdx.x) * EPL + r] = m[r];
            }
            for (int pp = 0; pp < 2 * K; ++pp) {
#pragma unroll
                for (int r = 0; r < EPL; ++r)
                    if (own[r]) buf[e[r]] = m[r];
                __syncwarp();
                float s[EPL];
#pragma unroll
                for (int r = 0; r < EPL; ++r) {
                    float acc = 0.0f;
#pragma unroll
                    for (int k = 0; k < N; ++k)
                        acc = __fadd_rn(acc, (pp & 1) == 0 ? buf[row[r] * N + k] : buf[k * N + col[r]]);
                    s[r] = acc;
                }
                __syncwarp();
#pragma unroll
                for (int r = 0; r < EPL; ++r) {
                    m[r] = __fdiv_rn(m[r], s[r]);
                    hist[((int64_t)(pp + 1) * blockDim.x + threadIdx.x) * EPL + r] = m[r];
                }
            }
            for (int pp = 2 * K - 1; pp >= 0; --pp) {
                float in[EPL], out[EPL];
#pragma unroll
                for (int r = 0; r < EPL; ++r) {
                    in[r] = hist[((int64_t)pp * blockDim.x + threadIdx.x) * EPL + r];
                    out[r] = hist[((int64_t)(pp + 1) * blockDim.x + threadIdx.x) * EPL + r];
                    if (own[r]) {
                        buf[e[r]] = in[r];
                        buf2[e[r]] = __fmul_rn(g[r], out[r]);
                    }
                }
                __syncwarp();
                float s[EPL], u[EPL];
#pragma unroll
                for (int r = 0; r < EPL; ++r) {
                    float as = 0.0f, au = 0.0f;
#pragma unroll
                    for (int k = 0; k < N; ++k) {
                        const int idx = (pp & 1) == 0 ? row[r] * N + k : k * N + col[r];
                        as = __fadd_rn(as, buf[idx]);
                        au = __fadd_rn(au, buf2[idx]);
                    }
                    s[r] = as;
                    u[r] = au;
                }
                __syncwarp();
#pragma unroll
                for (int r = 0; r < EPL; ++r) g[r] = __fdiv_rn(__fsub_rn(g[r], u[r]), s[r]);
            }
#pragma unroll
            for (int r = 0; r < EPL; ++r) {
                const float m0 = hist[((int64_t)0 * blockDim.x + threadIdx.x) * EPL + r];
                if (live && own[r]) dA[t * NN + e[r]] = __fmul_rn(g[r], m0);
            }
        }
        if (read) {
            // a = softmax(l) as the forward computes it, then dl = a (da - sum a da)
            float lq = (live && q < N) ? l[t * l_s + q] : 0.0f;
            float gq = (live && q < N) ? da[t * N + q] : 0.0f;
            const float aq = group_softmax<N>(lq, sw[warp], lane);
            float *ab = buf2;
            if (q < N) ab[q] = __fmul_rn(aq, gq);
            __syncwarp();
            float tsum = 0.0f;
#pragma unroll
            for (int k = 0; k < N; ++k) tsum = __fadd_rn(tsum, ab[k]);
            __syncwarp();
            if (live && q < N) da[t * N + q] = __fmul_rn(aq, __fsub_rn(gq, tsum));
        }
    }
}

// Block of 256 threads = 32 columns x 8 row slices: slice q sums rows
// q, q + 8, ... of its column in fp64, then the 8 partials are added in slice
// order. The order is fixed by the launch shape, so dg is reproducible.
constexpr int kDgCols = 32, kDgSlices = 8;
__global__ void __launch_bounds__(kDgCols * kDgSlices)
hc_dg_reduce_kernel(const float *part, int rows, int64_t d, float *dg) {
    __shared__ double acc_s[kDgSlices][kDgCols];
    const int col = threadIdx.x % kDgCols, q = threadIdx.x / kDgCols;
    for (int64_t k0 = (int64_t)blockIdx.x * kDgCols; k0 < d; k0 += (int64_t)gridDim.x * kDgCols) {
        const int64_t k = k0 + col;
        double acc = 0.0;
        if (k < d)
            for (int r = q; r < rows; r += kDgSlices) acc += (double)part[(int64_t)r * d + k];
        acc_s[q][col] = acc;
        __syncthreads();
        if (q == 0 && k < d) {
            double tot = 0.0;
#pragma unroll
            for (int j = 0; j < kDgSlices; ++j) tot += acc_s[j][col];
            dg[k] = (float)tot;
        }
        __syncthreads();
    }
}

#ifndef HC_BW_RING
#define HC_BW_RING 3  // cp.async staging stages of the step kernel (0: none)
#endif

template <int N, typename S>
struct StepBw {
    static constexpr int VE = bw_vec_elems<S>(N);
    // Static shared memory of the step kernel, and the dynamic budget that
    // leaves room for two CTAs per SM up to n = 5 (228 KB per SM, 1 KB
    // reserved per CTA), one CTA above.
    static constexpr size_t kStatic = 4 * ((size_t)kBwTB * (N * N + 2 * N)) + 16 * (kBwThreads / 32) +
                                      4 * (kBwThreads / 32) * (size_t)(2 * N + N * N + N) +
                                      4 * (kBwThreads / 32) * (size_t)kGroupScratch;
    static constexpr size_t kSmemPerSm = 228 * 1024;
    static constexpr size_t kDynBudget =
        N <= 5 ? kSmemPerSm / 2 - 1024 - kStatic - 256 : (size_t)kSmemLimitLogits - kStatic - 1024;
    static constexpr int kRing = HC_BW_RING;
    static_assert(kRing == 0 || kRing >= 2, "two staging stages at least");
    static size_t park_bytes(int64_t d) { return (size_t)d * 4; }  // h, fp32
    static size_t ring_bytes(int NT) { return (size_t)kRing * (2 * N + 2) * NT * VE * sizeof(S); }
    // 0: nothing staged; 1: h parked; 2: h parked and the rows staged through
    // the cp.async ring -- the deepest that fits the budget.
    static int mode(int64_t d, int NT) {
        if (park_bytes(d) > kDynBudget) return 0;
        if (kRing > 0 && park_bytes(d) + ring_bytes(NT) <= kDynBudget) return 2;
        return 1;
    }
    static size_t dyn_bytes(int64_t d, int NT) {
        const int md = mode(d, NT);
        return (md >= 1 ? park_bytes(d) : 0) + (md == 2 ? ring_bytes(NT) : 0);
    }
    template <int MD>
    static auto kernel() {
        return hc_step_bwd_kernel<N, S, VE, (MD >= 1), (MD == 2 ? kRing : 0)>;
    }
    static hc_status shape(int64_t d, int &NT) {
        const int64_t nvec = d / VE;
        int64_t nt = nvec < kBwThreads ? nvec : kBwThreads;
        nt = (nt + 31) / 32 * 32;
        // a CTA size that divides the row's slices, when one is near the largest
        for (int64_t c = nt; c >= nt / 2 && c >= 32 && nvec >= kBwThreads; c -= 32)
            if (nvec % c == 0) {
                nt = c;
                break;
            }
        if (nt < 32) nt = 32;
        NT = (int)nt;
        return HC_OK;
    }
    template <int MD>
    static hc_status occupancy(int NT, size_t dyn, int &per_sm) {
        auto kern = kernel<MD>();
        cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)dyn);
        if (e != cudaSuccess) return set_error(HC_ERR_CUDA, "backward smem attribute: %s", cudaGetErrorString(e));
        e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, NT, dyn);
        if (e != cudaSuccess) return set_error(HC_ERR_CUDA, "occupancy query: %s", cudaGetErrorString(e));
        return HC_OK;
    }
    // The TMA-fed kernel (hc_backward_pipe.cuh): bf16, n <= 4, only when the
    // pipelined path is forced (hc_set_path), and when its token buffer, dH'
    // ring, parked H' and gain partial fit shared memory (checked with the
    // ring, so the choice does not depend on dH'). It reads exactly the
    // minimum from DRAM, but the staged step kernel measured faster at
    // T = 16384, n = 4, d = 7168 (0.99 against 1.19 ms), so the automatic
    // choice is the step kernel.
    static bool pipelined(int64_t T, int64_t d, bool want_dg, const LaunchCtx &ctx, BwPipeShape &ps) {
        (void)T;
        if constexpr (sizeof(S) != 2 || N > 4) {
            return false;
        } else {
            if (ctx.path != 1) return false;
            const int64_t ntile = (d + kBwpTile - 1) / kBwpTile;
            if (ntile > 64) return false;
            ps.ntile = (int)ntile;
            ps.gstages = kBwpGradStages;
            return bwp_smem_bytes<N>(ps.ntile, ps.gstages, want_dg) <= (int64_t)kSmemLimitLogits;
        }
    }
    // Launch shape; the grid is what the gain-gradient workspace is sized by.
    static hc_status plan(int64_t T, int64_t d, bool want_dg, const LaunchCtx &ctx, int &NT,
                          int64_t &grid) {
        BwPipeShape ps{};
        if (pipelined(T, d, want_dg, ctx, ps)) {
            NT = kBwpThreads;
            grid = ctx.sms < T ? ctx.sms : T;
            if (grid < 1) grid = 1;
            return HC_OK;
        }
        shape(d, NT);
        const size_t dyn = dyn_bytes(d, NT);
        if (dyn > (size_t)kSmemLimitLogits - 16 * 1024)
            return set_error(HC_ERR_UNSUPPORTED, "d = %lld too large for the backward", (long long)d);
        int per_sm = 0;
        const int md = mode(d, NT);
        HC_BW_TRY(md == 2 ? occupancy<2>(NT, dyn, per_sm)
                          : md == 1 ? occupancy<1>(NT, dyn, per_sm) : occupancy<0>(NT, dyn, per_sm));
        if (per_sm < 1) per_sm = 1;
        grid = (int64_t)ctx.sms * per_sm;
        if (grid > T) grid = T;
        if (grid < 1) grid = 1;
        return HC_OK;
    }
    static hc_status launch(const BackwardArgs &a, const LaunchCtx &ctx, cudaStream_t st) {
        // the Sinkhorn backward's iterates must fit shared memory: check before any launch
        int pthreads = 128;
        const int Kh = a.f.mix_logits ? a.f.K : 0;
        size_t hist = (size_t)(2 * Kh + 1) * pthreads * Group<N>::EPL * 4;
        if (hist > (size_t)kSmemLimitLogits - 4096) {
            pthreads = 32;
            hist = (size_t)(2 * Kh + 1) * pthreads * Group<N>::EPL * 4;
        }
        if (hist > (size_t)kSmemLimitLogits - 4096)
            return set_error(HC_ERR_UNSUPPORTED, "K = %d too large for the Sinkhorn backward", a.f.K);
        const bool want_dg = a.dg != nullptr;
        int NT = 0;
        int64_t grid = 0;
        HC_BW_TRY(plan(a.f.T, a.f.d, want_dg, ctx, NT, grid));
        BwPipeShape ps{};
        if (pipelined(a.f.T, a.f.d, want_dg, ctx, ps)) {
            if constexpr (sizeof(S) == 2 && N <= 4) {
                if (!a.dHout) ps.gstages = 0;
                const int64_t smem = bwp_smem_bytes<N>(ps.ntile, ps.gstages, want_dg);
                auto kern = hc_bwd_pipe_kernel<N>;
                static std::atomic<int> configured[64];  // largest opt-in so far, per device
                if (ctx.device < 0 || ctx.device >= 64)
                    return set_error(HC_ERR_UNSUPPORTED, "device ordinal %d >= 64", ctx.device);
                if (smem > configured[ctx.device].load()) {
                    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                                         (int)smem);
                    if (e != cudaSuccess)
                        return set_error(HC_ERR_CUDA, "backward smem attribute: %s", cudaGetErrorString(e));
                    configured[ctx.device].store((int)smem);
                }
                BwPipeParams pp{};
                pp.f = a.f;
                pp.dHout = a.dHout;
                pp.dx = a.dx;
                pp.dH = a.dH;
                pp.dy = a.dy;
                pp.gA = a.dA;
                pp.gb = a.db;
                pp.ga = a.da;
                pp.dg_part = want_dg ? static_cast<float *>(a.workspace) : nullptr;
                kern<<<(unsigned)grid, kBwpThreads, (size_t)smem, st>>>(pp, ps, ctx.fault);
                cudaError_t e = cudaGetLastError();
                if (e != cudaSuccess)
                    return set_error(HC_ERR_CUDA, "hc_bwd_pipe_kernel launch: %s", cudaGetErrorString(e));
                return launch_tail(a, ctx, st, grid, hist, pthreads);
            }
        }
        BwKernelParams bp{};
        bp.f = a.f;
        bp.dHout = a.dHout;
        bp.dx = a.dx;
        bp.dH = a.dH;
        bp.dy = a.dy;
        bp.gA = a.dA;
        bp.gb = a.db;
        bp.ga = a.da;
        bp.dg_part = want_dg ? static_cast<float *>(a.workspace) : nullptr;
        const size_t dyn = dyn_bytes(a.f.d, NT);
        const int md = mode(a.f.d, NT);
        if (md == 2)
            kernel<2>()<<<(unsigned)grid, NT, dyn, st>>>(bp);
        else if (md == 1)
            kernel<1>()<<<(unsigned)grid, NT, dyn, st>>>(bp);
        else
            kernel<0>()<<<(unsigned)grid, NT, dyn, st>>>(bp);
        cudaError_t e = cudaGetLastError();
        if (e != cudaSuccess) return set_error(HC_ERR_CUDA, "hc_step_bwd_kernel launch: %s", cudaGetErrorString(e));
        return launch_tail(a, ctx, st, grid, hist, pthreads);
    }
    // The parameter backward (softmax, Sinkhorn) and the gain reduction over
    // the step kernel's `grid` partial rows.
    static hc_status launch_tail(const BackwardArgs &a, const LaunchCtx &ctx, cudaStream_t st,
                                 int64_t grid, size_t hist, int pthreads) {
        cudaError_t e;
        if (a.f.mix_logits || a.f.read_logits) {
            auto pk = hc_param_bwd_kernel<N>;
            e = cudaFuncSetAttribute(pk, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)hist);
            if (e != cudaSuccess) return set_error(HC_ERR_CUDA, "param backward smem: %s", cudaGetErrorString(e));
            const int64_t tok_per_block = (pthreads / 32) * Group<N>::TPW;
            int64_t pgrid = (a.f.T + tok_per_block - 1) / tok_per_block;
            if (pgrid > (int64_t)ctx.sms * 16) pgrid = (int64_t)ctx.sms * 16;
            pk<<<(unsigned)pgrid, pthreads, hist, st>>>(a.f.A, a.f.A_s, a.f.a, a.f.a_s, a.dA, a.da, a.f.T,
                                                        a.f.K, a.f.mix_logits, a.f.read_logits);
            e = cudaGetLastError();
            if (e != cudaSuccess) return set_error(HC_ERR_CUDA, "hc_param_bwd_kernel launch: %s", cudaGetErrorString(e));
        }
        if (a.dg) {
            int64_t rgrid = (a.f.d + kDgCols - 1) / kDgCols;
            if (rgrid > 4096) rgrid = 4096;
            hc_dg_reduce_kernel<<<(unsigned)rgrid, kDgCols * kDgSlices, 0, st>>>(static_cast<const float *>(a.workspace),
                                                                (int)grid, a.f.d, a.dg);
            e = cudaGetLastError();
            if (e != cudaSuccess) return set_error(HC_ERR_CUDA, "hc_dg_reduce_kernel launch: %s", cudaGetErrorString(e));
        }
        return HC_OK;
    }
};

template <typename S>
hc_status dispatch_bw_grid(int n, int64_t T, int64_t d, const LaunchCtx &ctx, int64_t &grid) {
    int NT = 0;
    switch (n) {
        case 1: return StepBw<1, S>::plan(T, d, true, ctx, NT, grid);
        case 2: return StepBw<2, S>::plan(T, d, true, ctx, NT, grid);
        case 3: return StepBw<3, S>::plan(T, d, true, ctx, NT, grid);
        case 4: return StepBw<4, S>::plan(T, d, true, ctx, NT, grid);
        case 5: return StepBw<5, S>::plan(T, d, true, ctx, NT, grid);
        case 6: return StepBw<6, S>::plan(T, d, true, ctx, NT, grid);
        case 7: return StepBw<7, S>::plan(T, d, true, ctx, NT, grid);
        default: return StepBw<8, S>::plan(T, d, true, ctx, NT, grid);
    }
}

template <typename S>
hc_status dispatch_bw(const BackwardArgs &a, const LaunchCtx &ctx, cudaStream_t st) {
    switch (a.n) {
        case 1: return StepBw<1, S>::launch(a, ctx, st);
        case 2: return StepBw<2, S>::launch(a, ctx, st);
        case 3: return StepBw<3, S>::launch(a, ctx, st);
        case 4: return StepBw<4, S>::launch(a, ctx, st);
        case 5: return StepBw<5, S>::launch(a, ctx, st);
        case 6: return StepBw<6, S>::launch(a, ctx, st);
        case 7: return StepBw<7, S>::launch(a, ctx, st);
        default: return StepBw<8, S>::launch(a, ctx, st);
    }
}

}  // namespace

hc_status backward_workspace_bytes(int n, hc_dtype dt, int64_t T, int64_t d, const LaunchCtx &ctx,
                                   size_t *bytes) {
    int64_t grid = 0;
    hc_status s = dt == HC_BF16 ? dispatch_bw_grid<__nv_bfloat16>(n, T, d, ctx, grid)
                                : dispatch_bw_grid<float>(n, T, d, ctx, grid);
    if (s != HC_OK) return s;
    *bytes = (size_t)grid * (size_t)d * sizeof(float);
    return HC_OK;
}

hc_status launch_backward(const BackwardArgs &a, const LaunchCtx &ctx, cudaStream_t st) {
    if (a.dg) {
        size_t need = 0;
        hc_status s = backward_workspace_bytes(a.n, a.dt, a.f.T, a.f.d, ctx, &need);
        if (s != HC_OK) return s;
        if (a.workspace_bytes < need)
            return set_error(HC_ERR_INVALID_ARG, "workspace of %zu bytes < %zu needed for dg",
                             a.workspace_bytes, need);
    }
    return a.dt == HC_BF16 ? dispatch_bw<__nv_bfloat16>(a, ctx, st) : dispatch_bw<float>(a, ctx, st);
}

}  // namespace hc
