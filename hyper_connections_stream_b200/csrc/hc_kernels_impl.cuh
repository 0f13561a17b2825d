// hc_kernels_impl.cuh -- launch-shape selection and dispatch over n for the
// step kernels. Included by one translation unit per (dtype, kind).
//
// Kernel families:
//   pipelined (hc_pipe_kernels.cuh): TMA-fed ring, warp-specialised; used
//     whenever at least two ring stages fit in shared memory next to the
//     groups' fp32 rows of h (normalising kinds);
//   register-streaming (hc_stream_kernels.cuh): no shared-memory staging;
//     covers the larger d of the normalising kinds and small (decode-sized)
//     calls, and can be forced.
#pragma once

#include <atomic>

#include "hc_launch.h"
#include "hc_pipe_kernels.cuh"
#include "hc_stream_kernels.cuh"

namespace hc {

// ---- register-streaming family ------------------------------------------------

template <int N, typename S, int KIND, int CPT>
hc_status launch_stream_cpt(const StepParams &p, int NT, const LaunchCtx &ctx, cudaStream_t st) {
    auto kern = hc_stream_kernel<N, S, KIND, CPT>;
    int per_sm = 0;
    cudaError_t e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, NT, 0);
    if (e != cudaSuccess) return set_error(HC_ERR_CUDA, "occupancy query: %s", cudaGetErrorString(e));
    if (per_sm < 1) per_sm = 1;
    int64_t grid = (int64_t)ctx.sms * per_sm;
    if (grid > p.T) grid = p.T;
    kern<<<(unsigned)grid, NT, 0, st>>>(p);
    e = cudaGetLastError();
    if (e != cudaSuccess) return set_error(HC_ERR_CUDA, "hc_stream_kernel launch: %s", cudaGetErrorString(e));
    return HC_OK;
}

// Threads per CTA (NT) and 16-byte slices per thread (CPT) for a row of nvec
// slices: the least idle slices, then the fewest slices per thread.
inline void pick_stream_shape(int64_t nvec, bool normalises, int &NT, int &CPT) {
    if (!normalises) {
        const int64_t t = nvec < 256 ? nvec : 256;
        NT = (int)((t + 31) / 32 * 32);
        CPT = 1;
        return;
    }
    static const int cpts[] = {1, 2, 4, 8};
    int best_nt = 0, best_cpt = 8;
    int64_t best_waste = INT64_MAX;
    for (int cpt : cpts) {
        int64_t nt = (nvec + cpt - 1) / cpt;
        nt = (nt + 31) / 32 * 32;
        if (nt > kStreamMaxThreads) continue;
        if (nt < 64 && cpt > 1) continue;
        const int64_t waste = nt * cpt - nvec;
        if (waste < best_waste) {
            best_waste = waste;
            best_nt = (int)nt;
            best_cpt = cpt;
        }
    }
    NT = best_nt;
    CPT = best_cpt;
}

template <int N, typename S, int KIND>
hc_status launch_stream(const StepParams &p, const LaunchCtx &ctx, cudaStream_t st) {
    constexpr int V = StorageTraits<S>::V;
    int NT = 0, CPT = 1;
    pick_stream_shape(p.d / V, kind_normalises(KIND), NT, CPT);
    if (NT == 0) return set_error(HC_ERR_UNSUPPORTED, "no launch shape for d = %lld", (long long)p.d);
    if constexpr (!kind_normalises(KIND)) {
        return launch_stream_cpt<N, S, KIND, 1>(p, NT, ctx, st);
    } else {
        switch (CPT) {
            case 1: return launch_stream_cpt<N, S, KIND, 1>(p, NT, ctx, st);
            case 2: return launch_stream_cpt<N, S, KIND, 2>(p, NT, ctx, st);
            case 4: return launch_stream_cpt<N, S, KIND, 4>(p, NT, ctx, st);
            default: return launch_stream_cpt<N, S, KIND, 8>(p, NT, ctx, st);
        }
    }
}

// ---- pipelined family -------------------------------------------------------------

// Ring geometry for a kind whose stages hold `rows` rows of a tile.
template <int N, typename S, int KIND, int GW = pipe_group_warps(N)>
bool pipe_shape(const StepParams &p, int rows, PipeShape &sh, int &smem) {
    constexpr int V = pipe_vec_elems<N, S>();
    const int64_t d_h = kind_normalises(KIND) ? p.d : 0;
    sh.tile = GW * 32 * V;
    const int64_t ntile = (p.d + sh.tile - 1) / sh.tile;
    if (ntile > (1 << 20)) return false;
    sh.ntile = (int)ntile;
    sh.stage_bytes = rows * sh.tile * (int)sizeof(S);
    // one ring per consumer group: the pipelined family needs room for two
    // stages per group; the ring then takes the kind's measured depth
    int64_t per_group = (kSmemLimit - pipe_fixed_bytes(N, 0, d_h, GW)) /
                        ((int64_t)kPipeGroups * (sh.stage_bytes + 16));
    if (per_group < 2) return false;
    if (per_group > kMaxStages / kPipeGroups) per_group = kMaxStages / kPipeGroups;
    const int64_t cap = KIND == KIND_WRITE ? HC_PIPE_SG_WRITE
                        : KIND == KIND_FUSED ? HC_PIPE_SG_FUSED
                        : KIND == KIND_REDUCE ? HC_PIPE_SG_REDUCE : HC_PIPE_SG_READ;
    if (per_group > cap) per_group = cap;
    if (per_group < 1) per_group = 1;
    sh.stages = (int)(per_group * kPipeGroups);
    smem = (int)((int64_t)sh.stages * sh.stage_bytes + pipe_fixed_bytes(N, sh.stages, d_h, GW));
    return true;
}

template <int N, typename S, int KIND, int GW = pipe_group_warps(N)>
bool pipe_shape(const StepParams &p, PipeShape &sh, int &smem) {
    return pipe_shape<N, S, KIND, GW>(p, KIND != KIND_READ ? N + 1 : N, sh, smem);
}

// The other consumer-group width a call may take: eight warps (576 threads;
// the compiler fits every kind in 96 registers without spills there), chosen
// when it pads the row's slices less than the default width does -- d =
// 4096 in bf16 is two tiles of 2048 instead of three of 1792. The read and
// write kinds take it up to n = 4 (static layer, T = 4096, n = 4, d = 4096:
// read 43.7 -> 40.7 us, write 52.4 -> 48.5 us); the fused and all-reduce
// kinds, whose consumers then run on fewer registers, at n <= 2 (n = 2,
// T = 16384: 71.7 -> 78.1 % of copy) and at n = 3, 4 only for calls of up to
// 8192 tokens (n = 4: T = 1024 +5 %, T = 4096 +3 %, but T = 16384 -1 %).
// Where seven-warp tiles fit exactly (d = 7168) the default stays.
template <int N, int KIND>
constexpr int pipe_alt_group_warps() { return N <= 4 ? 8 : pipe_group_warps(N); }

template <int N, typename S>
int64_t pipe_padded_slices(int64_t d, int gw) {
    const int64_t nvec = d / pipe_vec_elems<N, S>();
    const int64_t per = (int64_t)gw * 32;
    return (nvec + per - 1) / per * per;
}

template <int N, typename S, int KIND>
bool pipe_take_alt(int64_t d, int64_t T) {
    if constexpr (pipe_alt_group_warps<N, KIND>() == pipe_group_warps(N)) {
        return false;
    } else {
        if (!(KIND == KIND_READ || KIND == KIND_WRITE) && N > 2 && T > 8192) return false;
        return pipe_padded_slices<N, S>(d, pipe_alt_group_warps<N, KIND>()) <
               pipe_padded_slices<N, S>(d, pipe_group_warps(N));
    }
}

template <int N, typename S, int KIND, int GW = pipe_group_warps(N)>
hc_status launch_pipe(const StepParams &p, const PipeShape &sh, int smem, const LaunchCtx &ctx,
                      cudaStream_t st, const PipeReduce &rd = PipeReduce{}) {
    auto kern = hc_pipe_kernel<N, S, KIND, GW>;
    static std::atomic<int> configured[64];  // largest dynamic smem opted in so far, per device
    if (ctx.device < 0 || ctx.device >= 64)
        return set_error(HC_ERR_UNSUPPORTED, "device ordinal %d >= 64", ctx.device);
    if (smem > configured[ctx.device].load()) {
        cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
        if (e != cudaSuccess)
            return set_error(HC_ERR_CUDA, "cudaFuncSetAttribute(%d B smem): %s", smem,
                             cudaGetErrorString(e));
        configured[ctx.device].store(smem);
    }
    int64_t grid = ctx.sms;
    if (grid > p.T) grid = p.T;
    kern<<<(unsigned)grid, pipe_threads_gw(GW, pipe_param_warps(N)), smem, st>>>(p, sh, ctx.fault, rd);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return set_error(HC_ERR_CUDA, "hc_pipe_kernel launch: %s", cudaGetErrorString(e));
    return HC_OK;
}

// Which family a call takes (1 pipelined, 2 register-streaming), with the
// pipelined geometry when that family applies. From measurements of both
// (B200, bf16, graph-replayed calls, T = 256 ... 65536, n = 1 ... 8, d =
// 4096, 7168). The read kind: the register-streaming family at every size
// measured (5-39 % faster; within noise only at n = 3, 4, d = 7168). The
// write kind: register-streaming at n <= 2 (7-38 % faster), else below ~64
// MiB of stream traffic. The fused step: the pipeline needs enough tokens per
// CTA to amortise its fill and the first parameter batches -- a per-n token
// count (wider n: costlier Sinkhorn), times a factor when more than an eighth
// of the last seven-warp tile would idle (at n = 1 such rows stay
// register-streaming at any T: 6-10 % faster at d = 4096).
template <int N, typename S, int KIND>
int step_path_n(const StepParams &p, const LaunchCtx &ctx, bool &pipe_ok, bool &alt, PipeShape &sh,
                int &smem) {
    constexpr int GWA = pipe_alt_group_warps<N, KIND>();
    alt = pipe_take_alt<N, S, KIND>(p.d, p.T);
    pipe_ok = alt ? pipe_shape<N, S, KIND, GWA>(p, sh, smem) : pipe_shape<N, S, KIND>(p, sh, smem);
    bool small = p.T * (int64_t)N * p.d * (int64_t)sizeof(S) * 2 < (int64_t(64) << 20);
    if constexpr (KIND == KIND_READ) small = true;
    if constexpr (KIND == KIND_WRITE && N <= 2) small = true;
    if constexpr (KIND == KIND_FUSED) {
        constexpr int64_t tmin_n[9] = {0, 512, 512, 256, 256, 1024, 4096, 2048, 2048};
        constexpr int64_t ragged_x[9] = {0, int64_t(1) << 40, 64, 4, 4, 16, 4, 4, 4};
        // raggedness of the default width, which the thresholds were fitted on
        const int64_t nvec = p.d / pipe_vec_elems<N, S>();
        const int64_t slots = pipe_padded_slices<N, S>(p.d, pipe_group_warps(N));
        const bool ragged = (slots - nvec) * 8 > slots;
        small = p.T < tmin_n[N] * (ragged ? ragged_x[N] : 1);
    }
    return (ctx.path == 2 || !pipe_ok || (ctx.path == 0 && small)) ? 2 : 1;
}

template <int N, typename S, int KIND>
hc_status launch_step_n(const StepParams &p, const LaunchCtx &ctx, cudaStream_t st) {
    constexpr int GWA = pipe_alt_group_warps<N, KIND>();
    PipeShape sh{};
    int smem = 0;
    bool pipe_ok = false, alt = false;
    const int path = step_path_n<N, S, KIND>(p, ctx, pipe_ok, alt, sh, smem);
    if (ctx.path == 1 && !pipe_ok)
        return set_error(HC_ERR_UNSUPPORTED, "pipelined kernels do not cover d = %lld here",
                         (long long)p.d);
    if (path == 2) {
        if (kind_normalises(KIND) && p.d > (int64_t)kStreamMaxThreads * 8 * StorageTraits<S>::V)
            return set_error(HC_ERR_UNSUPPORTED, "d = %lld too large", (long long)p.d);
        return launch_stream<N, S, KIND>(p, ctx, st);
    }
    if (alt) return launch_pipe<N, S, KIND, GWA>(p, sh, smem, ctx, st);
    return launch_pipe<N, S, KIND>(p, sh, smem, ctx, st);
}

template <int N, typename S, int KIND>
hc_status launch_n(const StepParams &p, const LaunchCtx &ctx, cudaStream_t st) {
    if constexpr (KIND >= KIND_EXPAND) {
        // the ends of a stack run once per pass: register-streaming family only
        if (kind_normalises(KIND) && p.d > (int64_t)kStreamMaxThreads * 8 * StorageTraits<S>::V)
            return set_error(HC_ERR_UNSUPPORTED, "d = %lld too large", (long long)p.d);
        return launch_stream<N, S, KIND>(p, ctx, st);
    } else {
        return launch_step_n<N, S, KIND>(p, ctx, st);
    }
}

// ---- the fused all-reduce write (KIND_REDUCE), pipelined ------------------------

template <int N, typename S>
hc_status launch_reduce_pipe_n(const ReduceWriteArgs &ra, const bool *local, const LaunchCtx &ctx,
                               cudaStream_t st, bool *fits) {
    static_assert(kPipeMaxRanks == kMaxRanks, "rank limits agree");
    PipeReduce rd{};
    int nlocal = 0;
    for (int r = 0; r < kPipeMaxRanks; ++r) {
        rd.slot[r] = -1;
        if (r < ra.R) {
            rd.parts[r] = ra.parts[r];
            if (local[r]) rd.slot[r] = N + nlocal++;
        }
        if (r < ra.nx) rd.xs[r] = ra.xs[r];
    }
    rd.R = ra.R;
    rd.nx = ra.nx;
    rd.nlocal = nlocal;
    rd.y_out = ra.y_out;
    rd.t0 = ra.t0;
    PipeShape sh{};
    int smem = 0;
    constexpr int GWA = pipe_alt_group_warps<N, KIND_REDUCE>();
    const bool alt = pipe_take_alt<N, S, KIND_REDUCE>(ra.f.d, ra.f.T);
    *fits = alt ? pipe_shape<N, S, KIND_REDUCE, GWA>(ra.f, N + nlocal, sh, smem)
                : pipe_shape<N, S, KIND_REDUCE>(ra.f, N + nlocal, sh, smem);
    if (!*fits) return HC_OK;
    if (alt) return launch_pipe<N, S, KIND_REDUCE, GWA>(ra.f, sh, smem, ctx, st, rd);
    return launch_pipe<N, S, KIND_REDUCE>(ra.f, sh, smem, ctx, st, rd);
}

template <typename S>
hc_status launch_reduce_pipe(const ReduceWriteArgs &ra, const bool *local, const LaunchCtx &ctx,
                             cudaStream_t st, bool *fits) {
    switch (ra.n) {
        case 1: return launch_reduce_pipe_n<1, S>(ra, local, ctx, st, fits);
        case 2: return launch_reduce_pipe_n<2, S>(ra, local, ctx, st, fits);
        case 3: return launch_reduce_pipe_n<3, S>(ra, local, ctx, st, fits);
        case 4: return launch_reduce_pipe_n<4, S>(ra, local, ctx, st, fits);
        case 5: return launch_reduce_pipe_n<5, S>(ra, local, ctx, st, fits);
        case 6: return launch_reduce_pipe_n<6, S>(ra, local, ctx, st, fits);
        case 7: return launch_reduce_pipe_n<7, S>(ra, local, ctx, st, fits);
        default: return launch_reduce_pipe_n<8, S>(ra, local, ctx, st, fits);
    }
}

// The family launch_kind<S, KIND> would take for p (no launch).
template <typename S, int KIND>
int step_path(int n, const StepParams &p, const LaunchCtx &ctx) {
    if constexpr (KIND >= KIND_EXPAND) {
        return 2;
    } else {
        PipeShape sh{};
        int smem = 0;
        bool ok = false, alt = false;
        switch (n) {
            case 1: return step_path_n<1, S, KIND>(p, ctx, ok, alt, sh, smem);
            case 2: return step_path_n<2, S, KIND>(p, ctx, ok, alt, sh, smem);
            case 3: return step_path_n<3, S, KIND>(p, ctx, ok, alt, sh, smem);
            case 4: return step_path_n<4, S, KIND>(p, ctx, ok, alt, sh, smem);
            case 5: return step_path_n<5, S, KIND>(p, ctx, ok, alt, sh, smem);
            case 6: return step_path_n<6, S, KIND>(p, ctx, ok, alt, sh, smem);
            case 7: return step_path_n<7, S, KIND>(p, ctx, ok, alt, sh, smem);
            default: return step_path_n<8, S, KIND>(p, ctx, ok, alt, sh, smem);
        }
    }
}

template <typename S, int KIND>
hc_status launch_kind(int n, const StepParams &p, const LaunchCtx &ctx, cudaStream_t st) {
    switch (n) {
        case 1: return launch_n<1, S, KIND>(p, ctx, st);
        case 2: return launch_n<2, S, KIND>(p, ctx, st);
        case 3: return launch_n<3, S, KIND>(p, ctx, st);
        case 4: return launch_n<4, S, KIND>(p, ctx, st);
        case 5: return launch_n<5, S, KIND>(p, ctx, st);
        case 6: return launch_n<6, S, KIND>(p, ctx, st);
        case 7: return launch_n<7, S, KIND>(p, ctx, st);
        default: return launch_n<8, S, KIND>(p, ctx, st);
    }
}

}  // namespace hc
