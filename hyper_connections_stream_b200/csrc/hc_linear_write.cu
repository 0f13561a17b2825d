// hc_linear_write.cu -- the block's output projection fused with the write mix.
//
//   y[t][c]  = rnd_bf16( sum_k X[t][k] * Wo[c][k] )      (tensor cores, fp32 accumulation)
//   H'[t][j] = sum_i A[i][j] H[t][i] + b_j y[t]          (fp32 FMA chain in stream order)
//
// so the block's output y never makes a round trip through HBM: it is rounded
// to bf16 exactly as a stored y would be and consumed from the accumulator.
// (Hy4-preview model techniques map, models.inteligile.com: "inference
// kernel: kernel fusion used"; the glossary entry "Hyper-connections (mHC)":
// the streams are mixed after each block.)
//
// Persistent kernel, one CTA per SM, 192 threads; output tiles of 128 tokens x
// 256 channels are handed out round-robin:
//   warp 0      TMA producer: per k-step of 64, the 128B-swizzled X tile
//               (128 x 64) and Wo tile (256 x 64) into a ring of stages;
//   warp 1      allocates 512 TMEM columns (two 128 x 256 fp32 accumulators);
//               one lane issues tcgen05.mma (M = 128, N = 256, K = 16) and
//               commits each stage back to the producer and each finished
//               accumulator to the epilogue;
//   warps 2-5   epilogue, one thread per token row (TMEM lane): tcgen05.ld 16
//               channels of y, round to bf16, then for each 8-channel half
//               load the token's n stream slices, mix, store H'. The epilogue
//               of tile i overlaps the MMAs of tile i+1 (the other
//               accumulator).
// Every wait is bounded; on time-out the CTA records a fault, drains its
// copies and MMAs, frees TMEM and exits.
#include <cuda.h>

#include "hc_launch.h"
#include "hc_tc.cuh"

namespace hc {

namespace {

constexpr int kLwThreads = 192;
constexpr int kLwM = 128;                    // tokens per tile (TMEM lanes)
constexpr int kLwN = 256;                    // channels per tile (MMA N)
constexpr int kLwK = 64;                     // k per stage: one 128-byte swizzle row
constexpr int kLwABytes = kLwM * kLwK * 2;   // 16 KB
constexpr int kLwBBytes = kLwN * kLwK * 2;   // 32 KB
constexpr int kLwStageBytes = kLwABytes + kLwBBytes;
constexpr int kLwStages = 4;
constexpr uint32_t kLwTmemCols = 2 * kLwN;
constexpr int kLwSmem = 1024 /* alignment slack */ + kLwStages * kLwStageBytes +
                        (2 * kLwStages + 5) * 8 + 16;

struct LinearWriteParams {
    const __nv_bfloat16 *H;
    __nv_bfloat16 *Hout;
    __nv_bfloat16 *y;  // nullable
    const float *A;
    int64_t A_s;
    const float *b;
    int64_t b_s;
    int64_t T, d;
    int64_t tiles;
    int num_n;  // channel tiles
    int nk;     // k-steps per tile
};

__device__ __forceinline__ void load_bf16x8(const __nv_bfloat16 *p, float (&v)[8]) {
    const uint4 q = *reinterpret_cast<const uint4 *>(p);
    widen_bf16x2(q.x, v[0], v[1]);
    widen_bf16x2(q.y, v[2], v[3]);
    widen_bf16x2(q.z, v[4], v[5]);
    widen_bf16x2(q.w, v[6], v[7]);
}

__device__ __forceinline__ void store_bf16x8(__nv_bfloat16 *p, const float (&v)[8]) {
    uint4 q;
    q.x = pack_bf16x2_rn(v[0], v[1]);
    q.y = pack_bf16x2_rn(v[2], v[3]);
    q.z = pack_bf16x2_rn(v[4], v[5]);
    q.w = pack_bf16x2_rn(v[6], v[7]);
    *reinterpret_cast<uint4 *>(p) = q;
}

template <int N>
__global__ void __launch_bounds__(kLwThreads, 1)
hc_linear_write_kernel(const __grid_constant__ CUtensorMap mapX,
                       const __grid_constant__ CUtensorMap mapW, LinearWriteParams p, int *fault) {
    extern __shared__ __align__(1024) unsigned char smem_raw[];
    unsigned char *smem = reinterpret_cast<unsigned char *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    constexpr int S = kLwStages;
    uint64_t *full = reinterpret_cast<uint64_t *>(smem + S * kLwStageBytes);
    uint64_t *empty = full + S;
    uint64_t *acc_full = empty + S;      // [2]
    uint64_t *acc_empty = acc_full + 2;  // [2]
    uint64_t *drained = acc_empty + 2;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(drained + 1);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_slot + 1);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;

    if (threadIdx.x == 0) {
        for (int s = 0; s < S; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);  // the MMA commit
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(&acc_full[b], 1);   // the MMA commit
            mbar_init(&acc_empty[b], 4);  // the four epilogue warps
        }
        mbar_init(drained, 1);
        *abort_flag = 0;
        fence_barrier_init();
        prefetch_tensor_map(&mapX);
        prefetch_tensor_map(&mapW);
    }
    if (warp == 1) {
        tmem_alloc(tmem_slot, kLwTmemCols);
        tmem_relinquish();
    }
    tc_fence_before_sync();
    __syncthreads();
    tc_fence_after_sync();
    const uint32_t tmem = *tmem_slot;

    if (warp == 0) {
        // ---------------- TMA producer ----------------
        if (lane == 0) {
            int s = 0;
            uint32_t ph = 0;
            int64_t it = 0;
            bool ok = true;
            for (int64_t tile = blockIdx.x; ok && tile < p.tiles; tile += gridDim.x) {
                const int32_t m0 = (int32_t)(tile / p.num_n) * kLwM;
                const int32_t n0 = (int32_t)(tile % p.num_n) * kLwN;
                for (int ks = 0; ks < p.nk; ++ks, ++it) {
                    if (it >= S &&
                        !mbar_wait_bounded(&empty[s], ph ^ 1u, abort_flag, fault, FAULT_WAIT_EMPTY)) {
                        ok = false;
                        break;
                    }
                    unsigned char *st = smem + s * kLwStageBytes;
                    mbar_arrive_expect_tx(&full[s], (uint32_t)kLwStageBytes);
                    tma_load_2d(st, &mapX, ks * kLwK, m0, &full[s]);
                    tma_load_2d(st + kLwABytes, &mapW, ks * kLwK, n0, &full[s]);
                    if (++s == S) {
                        s = 0;
                        ph ^= 1u;
                    }
                }
            }
            // the copies still in flight land before the CTA exits
            for (int64_t q = (it > S ? it - S : 0); q < it; ++q)
                mbar_wait_drain(&full[q % S], (uint32_t)((q / S) & 1), fault);
        }
        __syncwarp();
    } else if (warp == 1) {
        // ---------------- MMA issuer ----------------
        if (lane == 0) {
            const uint32_t idesc = umma_idesc_bf16_f32(kLwM, kLwN);
            int s = 0;
            uint32_t ph = 0;
            int lt = 0;
            bool ok = true;
            for (int64_t tile = blockIdx.x; ok && tile < p.tiles; tile += gridDim.x, ++lt) {
                const int buf = lt & 1;
                if (lt >= 2 && !mbar_wait_bounded(&acc_empty[buf], (uint32_t)(((lt >> 1) & 1) ^ 1),
                                                  abort_flag, fault, FAULT_WAIT_REDUCE))
                    break;
                tc_fence_after_sync();
                const uint32_t dacc = tmem + (uint32_t)(buf * kLwN);
                for (int ks = 0; ks < p.nk; ++ks) {
                    if (!mbar_wait_bounded(&full[s], ph, abort_flag, fault, FAULT_WAIT_FULL)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after_sync();
                    const uint32_t a0 = smem_addr(smem + s * kLwStageBytes);
                    const uint32_t b0 = a0 + (uint32_t)kLwABytes;
#pragma unroll
                    for (int kk = 0; kk < kLwK / 16; ++kk) {
                        // +32 bytes along K per 16-element step inside the swizzle atom
                        umma_bf16(dacc, umma_desc_sw128(a0 + kk * 32), umma_desc_sw128(b0 + kk * 32),
                                  idesc, (ks | kk) != 0);
                    }
                    umma_commit(&empty[s]);  // stage free once these MMAs have read it
                    if (++s == S) {
                        s = 0;
                        ph ^= 1u;
                    }
                }
                if (!ok) break;
                umma_commit(&acc_full[buf]);  // accumulator complete
            }
            umma_commit(drained);  // every MMA issued so far has finished
            mbar_wait_drain(drained, 0, fault);
        }
        __syncwarp();
    } else {
        // ---------------- epilogue (warps 2..5) ----------------
        const int quarter = warp & 3;  // TMEM lanes this warp may access
        const int r = quarter * 32 + lane;
        const uint32_t lane_base = tmem + ((uint32_t)(quarter * 32) << 16);
        float Am[N][N], bv[N];
        if (p.A_s == 0) {
#pragma unroll
            for (int i = 0; i < N; ++i)
#pragma unroll
                for (int j = 0; j < N; ++j) Am[i][j] = p.A[i * N + j];
        }
        if (p.b_s == 0) {
#pragma unroll
            for (int j = 0; j < N; ++j) bv[j] = p.b[j];
        }
        int lt = 0;
        for (int64_t tile = blockIdx.x; tile < p.tiles; tile += gridDim.x, ++lt) {
            const int buf = lt & 1;
            const bool w = mbar_wait_bounded(&acc_full[buf], (uint32_t)((lt >> 1) & 1), abort_flag,
                                             fault, FAULT_WAIT_FULL);
            if (!__all_sync(0xffffffffu, w)) break;
            tc_fence_after_sync();
            const int64_t t = (tile / p.num_n) * kLwM + r;
            const int64_t n0 = (tile % p.num_n) * kLwN;
            const bool live = t < p.T;
            if (live) {
                if (p.A_s != 0) {
#pragma unroll
                    for (int i = 0; i < N; ++i)
#pragma unroll
                        for (int j = 0; j < N; ++j) Am[i][j] = p.A[t * p.A_s + i * N + j];
                }
                if (p.b_s != 0) {
#pragma unroll
                    for (int j = 0; j < N; ++j) bv[j] = p.b[t * p.b_s + j];
                }
            }
            const __nv_bfloat16 *Ht = p.H + t * N * p.d;
            __nv_bfloat16 *Hot = p.Hout + t * N * p.d;
            for (int c0 = 0; c0 < kLwN; c0 += 16) {
                uint32_t v[16];
                tmem_ld_32x32b_x16(lane_base + (uint32_t)(buf * kLwN + c0), v);
                tmem_ld_wait();
#pragma unroll
                for (int h = 0; h < 2; ++h) {
                    const int64_t c = n0 + c0 + 8 * h;
                    if (!live || c >= p.d) continue;
                    // y as a stored bf16 value would hold it
                    float yv[8];
#pragma unroll
                    for (int e = 0; e < 8; e += 2) {
                        const uint32_t q =
                            pack_bf16x2_rn(__uint_as_float(v[8 * h + e]), __uint_as_float(v[8 * h + e + 1]));
                        widen_bf16x2(q, yv[e], yv[e + 1]);
                    }
                    if (p.y) store_bf16x8(p.y + t * p.d + c, yv);
                    float hv[N][8];
#pragma unroll
                    for (int i = 0; i < N; ++i) load_bf16x8(Ht + i * p.d + c, hv[i]);
#pragma unroll
                    for (int j = 0; j < N; ++j) {
                        float acc[8];
#pragma unroll
                        for (int e = 0; e < 8; ++e) acc[e] = -0.0f;
#pragma unroll
                        for (int i = 0; i < N; ++i)
#pragma unroll
                            for (int e = 0; e < 8; ++e) acc[e] = __fmaf_rn(Am[i][j], hv[i][e], acc[e]);
#pragma unroll
                        for (int e = 0; e < 8; ++e) acc[e] = __fmaf_rn(bv[j], yv[e], acc[e]);
                        store_bf16x8(Hot + j * p.d + c, acc);
                    }
                }
            }
            tc_fence_before_sync();
            __syncwarp();
            if (lane == 0) mbar_arrive(&acc_empty[buf]);  // this accumulator may be refilled
        }
    }

    // every role has finished with TMEM (the MMA lane drained its MMAs)
    tc_fence_before_sync();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after_sync();
        tmem_dealloc(tmem, kLwTmemCols);
    }
}

template <int N>
hc_status launch_n_lw(const CUtensorMap &mapX, const CUtensorMap &mapW, const LinearWriteParams &lp,
                      const LaunchCtx &ctx, cudaStream_t st) {
    auto kern = hc_linear_write_kernel<N>;
    static bool configured[64] = {};
    if (ctx.device < 0 || ctx.device >= 64)
        return set_error(HC_ERR_UNSUPPORTED, "device ordinal %d >= 64", ctx.device);
    if (!configured[ctx.device]) {
        cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, kLwSmem);
        if (e != cudaSuccess)
            return set_error(HC_ERR_CUDA, "cudaFuncSetAttribute(%d B smem): %s", kLwSmem,
                             cudaGetErrorString(e));
        configured[ctx.device] = true;
    }
    int64_t grid = ctx.sms;
    if (grid > lp.tiles) grid = lp.tiles;
    kern<<<(unsigned)grid, kLwThreads, kLwSmem, st>>>(mapX, mapW, lp, ctx.fault);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess)
        return set_error(HC_ERR_CUDA, "hc_linear_write_kernel launch: %s", cudaGetErrorString(e));
    return HC_OK;
}

}  // namespace

hc_status launch_linear_write(const LinearWriteArgs &a, const LaunchCtx &ctx, cudaStream_t st) {
    static_assert(kLwSmem <= kSmemLimitLogits, "stages exceed the opt-in shared memory");
    LinearWriteParams lp{};
    lp.H = static_cast<const __nv_bfloat16 *>(a.H);
    lp.Hout = static_cast<__nv_bfloat16 *>(a.Hout);
    lp.y = static_cast<__nv_bfloat16 *>(a.y);
    lp.A = a.A;
    lp.A_s = a.A_s;
    lp.b = a.b;
    lp.b_s = a.b_s;
    lp.T = a.T;
    lp.d = a.d;
    const int64_t num_m = (a.T + kLwM - 1) / kLwM;
    const int64_t num_n = (a.d + kLwN - 1) / kLwN;
    const int64_t nk = (a.k + kLwK - 1) / kLwK;
    if (num_m > (int64_t(1) << 31) / kLwM || num_n > INT32_MAX || nk > INT32_MAX)
        return set_error(HC_ERR_UNSUPPORTED, "shape too large for the tile grid");
    lp.num_n = (int)num_n;
    lp.tiles = num_m * num_n;
    lp.nk = (int)nk;

    CUtensorMap mapX, mapW;
    hc_status ms = make_tma_map_bf16(&mapX, a.X, (uint64_t)a.k, (uint64_t)a.T, kLwK, kLwM);
    if (ms != HC_OK) return ms;
    ms = make_tma_map_bf16(&mapW, a.Wo, (uint64_t)a.k, (uint64_t)a.d, kLwK, kLwN);
    if (ms != HC_OK) return ms;
    switch (a.n) {
        case 1: return launch_n_lw<1>(mapX, mapW, lp, ctx, st);
        case 2: return launch_n_lw<2>(mapX, mapW, lp, ctx, st);
        case 3: return launch_n_lw<3>(mapX, mapW, lp, ctx, st);
        case 4: return launch_n_lw<4>(mapX, mapW, lp, ctx, st);
        case 5: return launch_n_lw<5>(mapX, mapW, lp, ctx, st);
        case 6: return launch_n_lw<6>(mapX, mapW, lp, ctx, st);
        case 7: return launch_n_lw<7>(mapX, mapW, lp, ctx, st);
        default: return launch_n_lw<8>(mapX, mapW, lp, ctx, st);
    }
}

}  // namespace hc
