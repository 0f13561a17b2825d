// hc_pipe_kernels.cuh -- warp-specialised, TMA-fed kernels of the HC step.
//
// One persistent CTA per SM (tokens blockIdx.x, blockIdx.x + G, ...) with
// threads in three roles:
//   warp 0      producer: one lane streams each token's n stream rows (and y)
//               tile by tile into shared-memory stages with plain bulk copies
//               (cp.async.bulk, this GPU's own memory, no multicast),
//               completing on the stage's "full" mbarrier;
//   warps 1..   parameters (pipe_param_warps(n) warps: one for n <= 5, more
//               for wider n, taking token batches round-robin): lane groups
//               compute the per-token Sinkhorn projection / read softmax
//               ahead of use into parameter slots;
//   the rest    consumer groups (kPipeGroups x pipe_group_warps(n) warps); group
//               r owns tokens r, r + kPipeGroups, ... of the CTA, reads the
//               stages, writes H' with coalesced 128-bit stores, keeps h in an
//               fp32 shared-memory row, reduces the fp64 sum of squares across
//               its warps, then stores x.
// KIND_REDUCE is the fused step with y the sum of R ranks' partial block
// outputs: a stage holds the n stream rows and the partial rows that are in
// this GPU's memory (bulk copies); partials in a peer's memory are read by
// the consumers with plain loads. The partials are added in rank order in
// fp32 and rounded once, so y is bit-identical on every rank.
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
#ifndef HC_PIPE_GROUP_WARPS_WIDE
#define HC_PIPE_GROUP_WARPS_WIDE 5
#endif
#ifndef HC_PIPE_L2_HINT
#define HC_PIPE_L2_HINT 0
#endif
// 1: the parameter warp projects its first batch with shuffle exchanges
// (shortest latency; the consumers wait on it), later batches through shared
// memory (highest throughput). Same results bit for bit either way.
#ifndef HC_PIPE_FIRST_SHFL
#define HC_PIPE_FIRST_SHFL 1
#endif
// Ring stages per consumer group, by kind. Shallow read-ahead keeps DRAM
// reads and writes balanced for the kinds that write as much as they read
// (measured on B200 at n = 4, d = 7168, bf16: write 2, fused 3); the read
// kind writes little and wants the deepest ring that fits.
#ifndef HC_PIPE_SG_WRITE
#define HC_PIPE_SG_WRITE 2
#endif
#ifndef HC_PIPE_SG_FUSED
#define HC_PIPE_SG_FUSED 3
#endif
#ifndef HC_PIPE_SG_READ
#define HC_PIPE_SG_READ 16
#endif
// The reduce kind reads R partial rows per tile besides the n stream rows.
#ifndef HC_PIPE_SG_REDUCE
#define HC_PIPE_SG_REDUCE 4
#endif
constexpr int kPipeGroups = HC_PIPE_GROUPS;
// Geometry for n > 5. Two Sinkhorn elements per lane and one token per warp
// make the projection cost about four times the instructions per token of
// n <= 5, and one parameter warp could not keep pace with the streams (at
// n = 6, d = 4096 the step ran at half the copy rate with K = 20 and at 88 %
// with K = 1). So several parameter warps share the token batches, and for
// n = 7, 8 the consumer groups narrow to four warps to keep the register
// budget (measured on B200: n = 6, d = 7168: 0.662 -> 0.600 ms; d = 4096:
// 0.593 -> 0.390 ms; n = 8, d = 4096: 0.688 -> 0.485 ms; n = 8, d = 7168
// within 1 %).
#ifndef HC_PIPE_GROUP_WARPS_6
#define HC_PIPE_GROUP_WARPS_6 5
#endif
#ifndef HC_PIPE_PARAM_WARPS_6
#define HC_PIPE_PARAM_WARPS_6 2
#endif
#ifndef HC_PIPE_GROUP_WARPS_78
#define HC_PIPE_GROUP_WARPS_78 4
#endif
#ifndef HC_PIPE_PARAM_WARPS_78
#define HC_PIPE_PARAM_WARPS_78 3
#endif
// Consumer warps per group: fewer for n > 4, so that each thread has the
// registers to hold n widened 16-byte rows (launch bounds give 65536 /
// threads registers a thread, the threads counted in whole 128-thread
// quarters: 128 at 16 warps, 170 at 12).
__host__ __device__ constexpr int pipe_group_warps(int n) {
    return n > 6 ? HC_PIPE_GROUP_WARPS_78 : n == 6 ? HC_PIPE_GROUP_WARPS_6
                 : n > 4 ? HC_PIPE_GROUP_WARPS_WIDE : HC_PIPE_GROUP_WARPS;
}
__host__ __device__ constexpr int pipe_param_warps(int n) {
    return n > 6 ? HC_PIPE_PARAM_WARPS_78 : n == 6 ? HC_PIPE_PARAM_WARPS_6 : 1;
}
__host__ __device__ constexpr int pipe_threads(int n) {
    return 32 * (1 + pipe_param_warps(n)) + kPipeGroups * pipe_group_warps(n) * 32;
}
// Threads of a pipelined CTA with gw consumer warps per group and npw
// parameter warps (plus the producer warp).
__host__ __device__ constexpr int pipe_threads_gw(int gw, int npw = 1) {
    return 32 * (1 + npw) + kPipeGroups * gw * 32;
}
// The parameter warp prepares kParamReplicas warps' worth of lane groups at a
// time (4 tokens for n = 3, 4; 2 for n >= 5); each group's slot ring holds at
// least 8 of its tokens, and two batches, so preparation runs ahead.
// Independent token batches the parameter warp runs through each Sinkhorn
// pass together (their latencies overlap).
constexpr int kParamReplicas = 2;
// n > 5 holds two matrix elements per lane and one token per warp, so its
// parameter warp runs four batches per pass to keep pace.
__host__ __device__ constexpr int pipe_param_replicas(int n) { return n > 5 ? 4 : kParamReplicas; }
__host__ __device__ constexpr int pipe_param_batch(int n) {
    return pipe_param_replicas(n) *
           (n * n <= 1 ? 32 : n * n <= 2 ? 16 : n * n <= 4 ? 8 : n * n <= 8 ? 4 : n * n <= 16 ? 2 : 1);
}
// Slots per group: at least 8 of its tokens, and one batch more than the
// parameter warps prepare at once, so preparation runs ahead.
__host__ __device__ constexpr int pipe_param_slots_per_group(int n) {
    return ((((pipe_param_warps(n) + 1) * pipe_param_batch(n) + kPipeGroups - 1) / kPipeGroups > 8
                 ? ((pipe_param_warps(n) + 1) * pipe_param_batch(n) + kPipeGroups - 1) / kPipeGroups
                 : 8) + 1) & ~1;  // even
}
constexpr int kMaxStages = 32;
constexpr int kSmemLimit = 232448;  // 227 KB opt-in dynamic shared memory per CTA

struct PipeShape {
    int stages;       // stages in all (kPipeGroups rings of stages / kPipeGroups)
    int tile;         // elements of d per tile (= group threads * pipe_vec_elems)
    int ntile;        // tiles per token
    int stage_bytes;  // bytes of one stage
};

// Extra arguments of KIND_REDUCE (unused by the other kinds).
constexpr int kPipeMaxRanks = 8;
struct PipeReduce {
    const void *parts[kPipeMaxRanks];  // partial y of each rank, rows t0 .. t0 + T - 1 used
    void *xs[kPipeMaxRanks];           // x_next destinations, same rows
    void *y_out;                       // reduced y [T][d] of this call's tokens, or null
    int64_t t0;                        // row of the partials and of x for token 0
    int R;                             // ranks
    int nx;                            // x destinations
    int nlocal;                        // partials staged by bulk copies
    int slot[kPipeMaxRanks];           // stage row of rank r's partial, -1: plain loads
};

// Bytes of everything in shared memory other than the ring: barriers,
// parameter slots, reduction partials, the abort flag and, for the
// normalising kinds, one fp32 row h[d] per group (d_h = d, else 0). The row
// serves two tokens at once: a thread reads back only its own slice
// positions, so at each tile it first reads the previous token's h there (for
// that token's x) and then overwrites it with the current token's.
__host__ __device__ constexpr int64_t pipe_fixed_bytes(int n, int stages, int64_t d_h,
                                                       int gw = -1) {
    return (int64_t)stages * 16                        // full + empty barriers
           + kPipeGroups * pipe_param_slots_per_group(n) * 16  // param full + empty
           + (kPipeGroups + 1) / 2 * 16                // group reduction barriers
           + kPipeGroups * pipe_param_slots_per_group(n) * (n * n + 2 * n) * 4  // slots
           + kPipeGroups * 2 * (gw > 0 ? gw : pipe_group_warps(n)) * 8  // reduction partials
           + 16                                        // abort flag (padded)
           + pipe_param_warps(n) * pipe_param_replicas(n) * kGroupScratch * 4  // parameter warps' scratch
           + (int64_t)kPipeGroups * ((d_h * 4 + 15) / 16 * 16);  // h rows (1 per group)
}


// Elements of d one consumer thread handles per tile: one 16-byte vector
// (n > 4 runs fewer, register-richer consumer threads to afford it), or with
// HC_PIPE_WIDE_HALF an 8-byte bf16 half vector for n > 4.
#ifndef HC_PIPE_WIDE_HALF
#define HC_PIPE_WIDE_HALF 0
#endif
template <int N, typename S>
__host__ __device__ constexpr int pipe_vec_elems() {
    return (HC_PIPE_WIDE_HALF && N > 4 && sizeof(S) == 2) ? 4 : StorageTraits<S>::V;
}

// Shared-memory loads and streaming global stores of VE storage elements,
// held as VE / 2 fp32 pairs (element 2p in .x, 2p + 1 in .y).
template <typename S, int VE> struct VecIO;
template <> struct VecIO<float, 4> {
    static __device__ __forceinline__ void load_smem(const unsigned char *p, float2 (&v)[2]) {
        const float4 q = *reinterpret_cast<const float4 *>(p);
        v[0] = make_float2(q.x, q.y);
        v[1] = make_float2(q.z, q.w);
    }
    static __device__ __forceinline__ void load_global(const float *p, float2 (&v)[2]) {
        const float4 q = __ldcs(reinterpret_cast<const float4 *>(p));
        v[0] = make_float2(q.x, q.y);
        v[1] = make_float2(q.z, q.w);
    }
    static __device__ __forceinline__ void round(float2 (&)[2]) {}
    static __device__ __forceinline__ void store(float *p, const float2 (&v)[2], float2 (&stored)[2]) {
        __stcs(reinterpret_cast<float4 *>(p), make_float4(v[0].x, v[0].y, v[1].x, v[1].y));
        stored[0] = v[0];
        stored[1] = v[1];
    }
    static __device__ __forceinline__ void store(float *p, const float2 (&v)[2]) {
        __stcs(reinterpret_cast<float4 *>(p), make_float4(v[0].x, v[0].y, v[1].x, v[1].y));
    }
};
__device__ __forceinline__ float2 widen_pair(uint32_t w) {
    float2 f;
    widen_bf16x2(w, f.x, f.y);
    return f;
}
template <> struct VecIO<__nv_bfloat16, 8> {
    static __device__ __forceinline__ void load_smem(const unsigned char *p, float2 (&v)[4]) {
        const uint4 q = *reinterpret_cast<const uint4 *>(p);
        v[0] = widen_pair(q.x);
        v[1] = widen_pair(q.y);
        v[2] = widen_pair(q.z);
        v[3] = widen_pair(q.w);
    }
    static __device__ __forceinline__ void load_global(const __nv_bfloat16 *p, float2 (&v)[4]) {
        const uint4 q = __ldcs(reinterpret_cast<const uint4 *>(p));
        v[0] = widen_pair(q.x);
        v[1] = widen_pair(q.y);
        v[2] = widen_pair(q.z);
        v[3] = widen_pair(q.w);
    }
    static __device__ __forceinline__ void round(float2 (&v)[4]) {
#pragma unroll
        for (int e = 0; e < 4; ++e) v[e] = widen_pair(pack_bf16x2_rn(v[e].x, v[e].y));
    }
    static __device__ __forceinline__ void store(__nv_bfloat16 *p, const float2 (&v)[4],
                                                 float2 (&stored)[4]) {
        uint4 q;
        q.x = pack_bf16x2_rn(v[0].x, v[0].y);
        q.y = pack_bf16x2_rn(v[1].x, v[1].y);
        q.z = pack_bf16x2_rn(v[2].x, v[2].y);
        q.w = pack_bf16x2_rn(v[3].x, v[3].y);
        __stcs(reinterpret_cast<uint4 *>(p), q);
        stored[0] = widen_pair(q.x);
        stored[1] = widen_pair(q.y);
        stored[2] = widen_pair(q.z);
        stored[3] = widen_pair(q.w);
    }
    static __device__ __forceinline__ void store(__nv_bfloat16 *p, const float2 (&v)[4]) {
        uint4 q;
        q.x = pack_bf16x2_rn(v[0].x, v[0].y);
        q.y = pack_bf16x2_rn(v[1].x, v[1].y);
        q.z = pack_bf16x2_rn(v[2].x, v[2].y);
        q.w = pack_bf16x2_rn(v[3].x, v[3].y);
        __stcs(reinterpret_cast<uint4 *>(p), q);
    }
};
template <> struct VecIO<__nv_bfloat16, 4> {
    static __device__ __forceinline__ void load_smem(const unsigned char *p, float2 (&v)[2]) {
        const uint2 q = *reinterpret_cast<const uint2 *>(p);
        v[0] = widen_pair(q.x);
        v[1] = widen_pair(q.y);
    }
    static __device__ __forceinline__ void load_global(const __nv_bfloat16 *p, float2 (&v)[2]) {
        const uint2 q = __ldcs(reinterpret_cast<const uint2 *>(p));
        v[0] = widen_pair(q.x);
        v[1] = widen_pair(q.y);
    }
    static __device__ __forceinline__ void round(float2 (&v)[2]) {
#pragma unroll
        for (int e = 0; e < 2; ++e) v[e] = widen_pair(pack_bf16x2_rn(v[e].x, v[e].y));
    }
    static __device__ __forceinline__ void store(__nv_bfloat16 *p, const float2 (&v)[2],
                                                 float2 (&stored)[2]) {
        uint2 q;
        q.x = pack_bf16x2_rn(v[0].x, v[0].y);
        q.y = pack_bf16x2_rn(v[1].x, v[1].y);
        __stcs(reinterpret_cast<uint2 *>(p), q);
        stored[0] = widen_pair(q.x);
        stored[1] = widen_pair(q.y);
    }
    static __device__ __forceinline__ void store(__nv_bfloat16 *p, const float2 (&v)[2]) {
        uint2 q;
        q.x = pack_bf16x2_rn(v[0].x, v[0].y);
        q.y = pack_bf16x2_rn(v[1].x, v[1].y);
        __stcs(reinterpret_cast<uint2 *>(p), q);
    }
};

// The n floats of a mixing-matrix column from a parameter slot, with the
// widest shared-memory loads the column's alignment allows (slots start on
// 16 bytes; a column starts at 4 n bytes into its slot): one LDS.128 per
// four values for n % 4 == 0, one LDS.64 per pair for even n.
template <int N>
__device__ __forceinline__ void load_column(const float *c, float (&col)[N]) {
    if constexpr (N % 4 == 0) {
#pragma unroll
        for (int q = 0; q < N; q += 4) {
            const float4 v = *reinterpret_cast<const float4 *>(c + q);
            col[q] = v.x; col[q + 1] = v.y; col[q + 2] = v.z; col[q + 3] = v.w;
        }
    } else if constexpr (N % 2 == 0) {
#pragma unroll
        for (int q = 0; q < N; q += 2) {
            const float2 v = *reinterpret_cast<const float2 *>(c + q);
            col[q] = v.x; col[q + 1] = v.y;
        }
    } else {
#pragma unroll
        for (int q = 0; q < N; ++q) col[q] = c[q];
    }
}

// The parameter warp of the pipelined kernels. Token m of the CTA (token
// blockIdx.x + m * G) belongs to consumer group m % NG as that group's token
// m / NG, whose parameters go to slot (m % NG) * PSG + (m / NG) % PSG of
// `params` (PSTRIDE = n*n + 2n floats: A transposed, column j at j * n, then
// b, then a), published on pfull and reclaimed through pempty (each with one
// arrival per use: this warp, resp. the group's consumer warps).
template <int N, bool WRITE, bool READ, int NG, int PSG>
__device__ __forceinline__ void pipe_param_warp(const StepParams &p, int64_t M, int64_t G, float *params,
                                                uint64_t *pfull, uint64_t *pempty, float *pscratch,
                                                volatile int *abort_flag, int *fault, int lane,
                                                int pw = 0, int npw = 1) {
    constexpr int NN = N * N;
    constexpr int PSTRIDE = NN + 2 * N;
    constexpr int PB = pipe_param_batch(N);
    // ---------------- per-token parameters ----------------
    // Batch replica rb, lane group lane / GL prepares token
    // m0 + rb * TPW + lane / GL. The next batch's inputs are loaded
    // before the current batch is projected, hiding their latency.
    constexpr int GL = Group<N>::GL, EPL = Group<N>::EPL, TPW = Group<N>::TPW;
    constexpr int R = pipe_param_replicas(N);
    static_assert(R * TPW == PB, "a batch is R warps' worth of lane groups");
    const int q = lane & (GL - 1);
    float nmv[R][EPL], nlv[R], nbv[R];
    auto fetch = [&](int64_t m0) {
#pragma unroll
        for (int rb = 0; rb < R; ++rb) {
            const int64_t m = m0 + rb * TPW + lane / GL;
            const bool live = m < M;
            const int64_t t = blockIdx.x + m * G;
#pragma unroll
            for (int r = 0; r < EPL; ++r) {
                const int e = q + GL * r;
                nmv[rb][r] = (WRITE && live && e < NN) ? p.A[t * p.A_s + e] : 0.0f;
            }
            nbv[rb] = (WRITE && live && q < N) ? p.b[t * p.b_s + q] : 0.0f;
            nlv[rb] = (READ && live && q < N) ? p.a[t * p.a_s + q] : 0.0f;
        }
    };
    // parameter warp pw of npw takes batches pw, pw + npw, ...
    fetch((int64_t)pw * PB);
    for (int64_t m0 = (int64_t)pw * PB; m0 < M; m0 += (int64_t)npw * PB) {
        float mv[R][EPL], lv[R], bvv[R];
#pragma unroll
        for (int rb = 0; rb < R; ++rb) {
#pragma unroll
            for (int r = 0; r < EPL; ++r) mv[rb][r] = nmv[rb][r];
            lv[rb] = nlv[rb];
            bvv[rb] = nbv[rb];
        }
        if (m0 + (int64_t)npw * PB < M) fetch(m0 + (int64_t)npw * PB);
        bool w = true;
#pragma unroll
        for (int rb = 0; rb < R; ++rb) {
            const int64_t m = m0 + rb * TPW + lane / GL;
            const int64_t i = m / NG;  // token ordinal within its group
            const int ps = (int)(m % NG) * PSG + (int)(i % PSG);
            if (m < M && i >= PSG)
                w = w && mbar_wait_bounded(&pempty[ps], (uint32_t)(((i / PSG) & 1) ^ 1), abort_flag,
                                           fault, FAULT_WAIT_PARAM);
        }
        if (!__all_sync(0xffffffffu, w)) break;
        if constexpr (WRITE) {
            if (p.mix_logits) {
                // the consumers wait on the first batch: project it with the
                // shortest-latency exchange (same results bit for bit)
                if (HC_PIPE_FIRST_SHFL && m0 < (int64_t)npw * PB)
                    group_sinkhorn<N, R, true>(mv, pscratch, lane, p.K);
                else
                    group_sinkhorn<N, R, false>(mv, pscratch, lane, p.K);
            }
        }
        if constexpr (READ) {
            if (p.read_logits) {
#pragma unroll
                for (int rb = 0; rb < R; ++rb) lv[rb] = group_softmax<N>(lv[rb], pscratch, lane);
            }
        }
#pragma unroll
        for (int rb = 0; rb < R; ++rb) {
            const int64_t m = m0 + rb * TPW + lane / GL;
            if (m >= M) continue;
            const int64_t i = m / NG;
            const int ps = (int)(m % NG) * PSG + (int)(i % PSG);
            float *P = params + ps * PSTRIDE;
            if constexpr (WRITE) {
#pragma unroll
                for (int r = 0; r < EPL; ++r) {
                    const int e = q + GL * r;  // A[i][j], i = e / N, j = e % N
                    if (e < NN) P[(e % N) * N + e / N] = mv[rb][r];
                }
                if (q < N) P[NN + q] = bvv[rb];
            }
            if constexpr (READ) {
                if (q < N) P[NN + N + q] = lv[rb];
            }
        }
        __syncwarp();
#pragma unroll
        for (int rb = 0; rb < R; ++rb) {
            const int64_t m = m0 + rb * TPW + lane / GL;
            if (m < M && q == 0) {
                const int64_t i = m / NG;
                mbar_arrive(&pfull[(int)(m % NG) * PSG + (int)(i % PSG)]);
            }
        }
    }
}

template <int N, typename S, int KIND, int GW = pipe_group_warps(N)>
__global__ void __launch_bounds__(pipe_threads_gw(GW, pipe_param_warps(N)), 1)
hc_pipe_kernel(StepParams p, PipeShape sh, int *fault, PipeReduce rd) {
    constexpr int V = pipe_vec_elems<N, S>();
    constexpr int VB = V * (int)sizeof(S);  // bytes per thread per row of a tile
    constexpr int NN = N * N;
    constexpr bool WRITE = KIND != KIND_READ;
    constexpr bool READ = KIND != KIND_WRITE;
    constexpr bool REDUCE = KIND == KIND_REDUCE;
    const int ROWS = REDUCE ? N + rd.nlocal : WRITE ? N + 1 : N;
    constexpr int PSTRIDE = NN + 2 * N;  // A transposed (column j at j*N) | b | a
    constexpr int NG = kPipeGroups;
    constexpr int PSG = pipe_param_slots_per_group(N);
    constexpr int kParamSlots = NG * PSG;
    constexpr int PB = pipe_param_batch(N);

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
    float *pscratch = reinterpret_cast<float *>(abort_word + 4);  // parameter warp scratch
    constexpr int NPW = pipe_param_warps(N);
    float *hrow_base = pscratch + NPW * pipe_param_replicas(N) * kGroupScratch;  // 16-byte aligned
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
        // per group ring: tiles issued, tiles to issue, and the ring position,
        // the phase and the (token ordinal, tile) of the next tile
        int64_t nq[NG], qend[NG], mr[NG];
        int slot_r[NG], tile_r[NG];
        uint32_t ph_r[NG];
#pragma unroll
        for (int r = 0; r < NG; ++r) {
            nq[r] = 0;
            qend[r] = (M > r ? (M - 1 - r) / NG + 1 : 0) * (int64_t)ntile;
            mr[r] = r;
            slot_r[r] = 0;
            tile_r[r] = 0;
            ph_r[r] = 0;
        }
        uint64_t idle_since = 0;
        uint32_t backoff = 32;
        [[maybe_unused]] const uint64_t policy = HC_PIPE_L2_HINT ? l2_policy_evict_first() : 0;
        auto load = [&](void *dst, const void *src, uint32_t bytes, uint64_t *bar) {
            if constexpr (HC_PIPE_L2_HINT) bulk_load_hint(dst, src, bytes, bar, policy);
            else bulk_load(dst, src, bytes, bar);
        };
        for (;;) {
            bool pending = false, progressed = false;
#pragma unroll
            for (int r = 0; r < NG; ++r) {
                if (nq[r] >= qend[r]) continue;
                pending = true;
                const int s = r * SG + slot_r[r];
                if (nq[r] >= SG && !mbar_test_wait(&empty[s], ph_r[r] ^ 1u)) continue;
                const int64_t t = blockIdx.x + mr[r] * G;
                const int64_t k0 = (int64_t)tile_r[r] * tile;
                const int64_t w = (d - k0) < tile ? (d - k0) : tile;
                const uint32_t rb = (uint32_t)(w * (int64_t)sizeof(S));
                unsigned char *st = ring + (size_t)s * sh.stage_bytes;
                mbar_arrive_expect_tx(&full[s], rb * ROWS);
                const S *src = H + t * N * d + k0;
#pragma unroll
                for (int i = 0; i < N; ++i) load(st + i * row_bytes, src + i * d, rb, &full[s]);
                if constexpr (REDUCE) {
                    const int64_t off = (rd.t0 + t) * d + k0;
#pragma unroll
                    for (int q = 0; q < kPipeMaxRanks; ++q)
                        if (q < rd.R && rd.slot[q] >= 0)
                            load(st + rd.slot[q] * row_bytes, static_cast<const S *>(rd.parts[q]) + off,
                                 rb, &full[s]);
                } else if constexpr (WRITE) {
                    load(st + N * row_bytes, Y + t * d + k0, rb, &full[s]);
                }
                ++nq[r];
                if (++slot_r[r] == SG) {
                    slot_r[r] = 0;
                    ph_r[r] ^= 1u;
                }
                if (++tile_r[r] == ntile) {
                    tile_r[r] = 0;
                    mr[r] += NG;
                }
                progressed = true;
            }
            if (!pending) break;
            if (progressed) {
                idle_since = 0;
                backoff = 32;
                continue;
            }
            // every ring is full: back off (up to ~1 us); give up only after the limit
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
#pragma unroll
        for (int r = 0; r < NG; ++r)
            for (int64_t qq = (nq[r] > SG ? nq[r] - SG : 0); qq < nq[r]; ++qq)
                mbar_wait_drain(&full[r * SG + (int)(qq % SG)], (uint32_t)((qq / SG) & 1), fault);
        return;
    }

    if (warp >= 1 && warp <= NPW) {
        pipe_param_warp<N, WRITE, READ, NG, PSG>(
            p, M, G, params, pfull, pempty, pscratch + (warp - 1) * pipe_param_replicas(N) * kGroupScratch,
            abort_flag, fault, lane, warp - 1, NPW);
        return;
    }

    // ---------------- consumers ----------------
    // Group g takes the CTA's tokens g, g + NG, ... (its i-th token is
    // m = g + i * NG). While it processes token i tile by tile, it also writes
    // token i-1's x, one tile after each of token i's tiles: a warp arrives at
    // the group reduction of token i-1 and goes on to token i's first tile
    // before it waits for the other warps' sums, so the wait overlaps work.
    // Both tokens share the group's h row: at each tile a thread reads token
    // i-1's h at its own slice positions before it stores token i's there.
    const int cw = warp - 1 - NPW;
    const int g = cw / GW;
    const int gw = cw - g * GW;
    const int gt = gw * 32 + lane;
    uint64_t *gfull = full + g * SG;
    uint64_t *gempty = empty + g * SG;
    unsigned char *gring = ring + (size_t)g * SG * sh.stage_bytes;
    float *hrow = hrow_base + g * hrow_stride;
    S *Ho = static_cast<S *>(p.Hout);
    S *X = static_cast<S *>(p.x);
    int slot = 0;      // ring position of this group's next tile
    uint32_t ph = 0;   // its phase parity
    const int64_t Mg = M > g ? (M - 1 - g) / NG + 1 : 0;  // tokens of this group
    float r_prev = 0.0f;
    constexpr int VP = V / 2;  // element pairs per thread

    for (int64_t i = 0; i <= Mg; ++i) {
        const bool cur = i < Mg;                 // token i to mix
        const bool prev = READ && i > 0;         // token i-1 to normalise
        const int64_t m = g + i * NG;
        const int64_t t = blockIdx.x + m * G;
        const int64_t t_prev = t - (int64_t)NG * G;
        const int ps = g * PSG + (int)(i % PSG);
        float bv[N], av[N];
        const float *P = params + ps * PSTRIDE;
        if (cur) {
            const bool w = mbar_wait_bounded(&pfull[ps], (uint32_t)((i / PSG) & 1), abort_flag, fault,
                                             FAULT_WAIT_PARAM);
            if (!__all_sync(0xffffffffu, w)) break;
#pragma unroll
            for (int ii = 0; ii < N; ++ii) {
                bv[ii] = WRITE ? P[NN + ii] : 0.0f;
                av[ii] = READ ? P[NN + N + ii] : 0.0f;
            }
        }

        bool ok = true;
        double ss = 0.0;
        for (int j = 0; j < ntile; ++j) {
            const int64_t k = (int64_t)j * tile + (int64_t)gt * V;
            const bool active = k < d;
            float2 hr[VP];  // token i's h at this thread's slice of tile j
            if (cur) {
                const int cs = slot;
                const bool w = mbar_wait_bounded(&gfull[cs], ph, abort_flag, fault, FAULT_WAIT_FULL);
                if (!__all_sync(0xffffffffu, w)) {
                    ok = false;
                    break;
                }
                if (++slot == SG) {
                    slot = 0;
                    ph ^= 1u;
                }
                const unsigned char *st = gring + (size_t)cs * sh.stage_bytes + (size_t)gt * VB;
                float2 h[N][VP], yv[VP];
                if (active) {
#pragma unroll
                    for (int ii = 0; ii < N; ++ii) VecIO<S, V>::load_smem(st + ii * row_bytes, h[ii]);
                    if constexpr (REDUCE) {
                        // the all-reduce of y: partials added in rank order
                        const int64_t off = (rd.t0 + t) * d + k;
#pragma unroll
                        for (int q = 0; q < kPipeMaxRanks; ++q) {
                            if (q < rd.R) {
                                float2 pv[VP];
                                if (rd.slot[q] >= 0)
                                    VecIO<S, V>::load_smem(st + rd.slot[q] * row_bytes, pv);
                                else
                                    VecIO<S, V>::load_global(static_cast<const S *>(rd.parts[q]) + off, pv);
                                if (q == 0) {
#pragma unroll
                                    for (int e = 0; e < VP; ++e) yv[e] = pv[e];
                                } else {
#pragma unroll
                                    for (int e = 0; e < VP; ++e) yv[e] = fadd2_rn(yv[e], pv[e]);
                                }
                            }
                        }
                    } else if constexpr (WRITE) {
                        VecIO<S, V>::load_smem(st + N * row_bytes, yv);
                    }
                }
                __syncwarp();
                if (lane == 0) mbar_arrive(&gempty[cs]);  // stage data is in registers
                if (active) {
                    if constexpr (REDUCE) {
                        // one rounding to the storage dtype (what a stored y holds)
                        if (rd.y_out) {
                            float2 stored[VP];
                            VecIO<S, V>::store(static_cast<S *>(rd.y_out) + t * d + k, yv, stored);
#pragma unroll
                            for (int e = 0; e < VP; ++e) yv[e] = stored[e];
                        } else {
                            VecIO<S, V>::round(yv);
                        }
                    }
                    if constexpr (WRITE) {
                        S *Hot = Ho + t * N * d + k;
#pragma unroll
                        for (int jj = 0; jj < N; ++jj) {
                            // column jj of A: A[0][jj] .. A[N-1][jj] (contiguous in the slot)
                            float col[N];
                            load_column<N>(P + jj * N, col);
                            float2 acc[VP], stored[VP];
                            const float2 c0 = make_float2(col[0], col[0]);
#pragma unroll
                            for (int e = 0; e < VP; ++e) acc[e] = fmul2_rn(c0, h[0][e]);
#pragma unroll
                            for (int ii = 1; ii < N; ++ii) {
                                const float2 ci = make_float2(col[ii], col[ii]);
#pragma unroll
                                for (int e = 0; e < VP; ++e) acc[e] = ffma2_rn(ci, h[ii][e], acc[e]);
                            }
                            const float2 cb = make_float2(bv[jj], bv[jj]);
#pragma unroll
                            for (int e = 0; e < VP; ++e) acc[e] = ffma2_rn(cb, yv[e], acc[e]);
                            VecIO<S, V>::store(Hot + jj * d, acc, stored);
                            if constexpr (READ) {
                                const float2 ca = make_float2(av[jj], av[jj]);
                                if (jj == 0) {
#pragma unroll
                                    for (int e = 0; e < VP; ++e) hr[e] = fmul2_rn(ca, stored[e]);
                                } else {
#pragma unroll
                                    for (int e = 0; e < VP; ++e) hr[e] = ffma2_rn(ca, stored[e], hr[e]);
                                }
                            }
                        }
                    } else {
                        const float2 c0 = make_float2(av[0], av[0]);
#pragma unroll
                        for (int e = 0; e < VP; ++e) hr[e] = fmul2_rn(c0, h[0][e]);
#pragma unroll
                        for (int ii = 1; ii < N; ++ii) {
                            const float2 ci = make_float2(av[ii], av[ii]);
#pragma unroll
                            for (int e = 0; e < VP; ++e) hr[e] = ffma2_rn(ci, h[ii][e], hr[e]);
                        }
                    }
                    if constexpr (READ) {
#pragma unroll
                        for (int e = 0; e < VP; ++e) {
                            const double hx = (double)hr[e].x, hy = (double)hr[e].y;
                            ss = __fma_rn(hx, hx, ss);
                            ss = __fma_rn(hy, hy, ss);
                        }
                    }
                }
            }
            if constexpr (READ) {
                if (prev) {
                    if (j == 0) {
                        // token i-1's sum of squares, reduced over the group's warps
                        const bool w = mbar_wait_bounded(&redbar[g], (uint32_t)((i - 1) & 1), abort_flag,
                                                         fault, FAULT_WAIT_REDUCE);
                        if (!__all_sync(0xffffffffu, w)) {
                            ok = false;
                            break;
                        }
                        const double *part = sred + (g * 2 + (int)((i - 1) & 1)) * GW;
                        double tot = 0.0;
#pragma unroll
                        for (int ii = 0; ii < GW; ++ii) tot += part[ii];
                        r_prev = __double2float_rn(1.0 / sqrt(tot / (double)d + (double)p.eps));
                    }
                    if (active) {
                        float gv[V];
                        float2 hv[VP], xv[VP];
                        load_gain<V>(p.g, k, gv);
#pragma unroll
                        for (int e = 0; e < VP; e += 2) {
                            const float4 f = *reinterpret_cast<const float4 *>(hrow + k + 2 * e);
                            hv[e] = make_float2(f.x, f.y);
                            hv[e + 1] = make_float2(f.z, f.w);
                        }
                        const float2 r2 = make_float2(r_prev, r_prev);
#pragma unroll
                        for (int e = 0; e < VP; ++e)
                            xv[e] = fmul2_rn(fmul2_rn(hv[e], r2), make_float2(gv[2 * e], gv[2 * e + 1]));
                        if constexpr (REDUCE) {
                            // x_next to every destination (the all-gather of the
                            // reduce-scatter form: peers' buffers take plain stores)
                            const int64_t off = (rd.t0 + t_prev) * d + k;
#pragma unroll
                            for (int q = 0; q < kPipeMaxRanks; ++q)
                                if (q < rd.nx) VecIO<S, V>::store(static_cast<S *>(rd.xs[q]) + off, xv);
                        } else {
                            VecIO<S, V>::store(X + t_prev * d + k, xv);
                        }
                    }
                }
                // keep token i's h for its normalisation (after token i-1's read above)
                if (cur && active) {
#pragma unroll
                    for (int e = 0; e < VP; e += 2)
                        *reinterpret_cast<float4 *>(hrow + k + 2 * e) =
                            make_float4(hr[e].x, hr[e].y, hr[e + 1].x, hr[e + 1].y);
                }
            }
        }
        if (!ok) break;
        if (cur) {
            __syncwarp();
            if (lane == 0) mbar_arrive(&pempty[ps]);  // parameters no longer read
            if constexpr (READ) {
#pragma unroll
                for (int off = 16; off > 0; off >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, off);
                if (lane == 0) {
                    sred[(g * 2 + (int)(i & 1)) * GW + gw] = ss;
                    mbar_arrive(&redbar[g]);
                }
            }
        }
    }
}

}  // namespace hc
