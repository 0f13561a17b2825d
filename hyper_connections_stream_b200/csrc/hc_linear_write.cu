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
// Persistent kernel on CTA pairs (clusters of two, one CTA per SM, 192
// threads each); output tiles of 256 tokens x 256 channels are handed out
// round-robin to the pairs. CTA r of a pair stages token rows 128r..128r+127
// of X and channel rows 128r..128r+127 of Wo, so each SM streams 32 KB per
// k-step for a 256 x 256 x 64 product (a third less than one CTA per tile):
//   warp 0      TMA producer: per k-step of 64, the 128B-swizzled X and Wo
//               halves into a ring of stages; the bytes of both CTAs complete
//               on the leader's stage barrier;
//   warp 1      TMEM (512 columns: two 128 x 256 fp32 accumulators per CTA,
//               allocated for the pair); in the leader one lane issues
//               tcgen05.mma.cta_group::2 (M = 256, N = 256, K = 16) and
//               commits each stage and each finished accumulator to both CTAs;
//   warps 2-5   epilogue of this CTA's 128 rows: tcgen05.ld of the
//               accumulator (one token row per thread), rounded to bf16 and
//               transposed through shared memory, then the write mix of the
//               token's n stream slices with coalesced 256-byte loads and
//               stores; the accumulator is handed back to the leader's MMA as
//               soon as it has been read, so the epilogue of tile i overlaps
//               the MMAs of tile i+1.
// Every wait is bounded; on time-out a CTA records a fault, drains its copies
// and MMAs and leaves through the closing cluster barrier.
#include <cuda.h>

#include <atomic>

#include "hc_launch.h"
#include "hc_tc.cuh"

namespace hc {

namespace {

constexpr int kLwThreads = 192;
constexpr int kLwM = 128;                    // token rows per CTA (TMEM lanes)
constexpr int kLwTileM = 2 * kLwM;           // token rows per pair tile (MMA M)
constexpr int kLwN = 256;                    // channels per tile (MMA N)
constexpr int kLwBRows = kLwN / 2;           // Wo rows staged per CTA
constexpr int kLwKSub = 64;                  // one 128-byte swizzle row
constexpr int kLwSubs = 2;                   // adjacent sub-tiles per stage
constexpr int kLwK = kLwKSub * kLwSubs;      // k per stage
constexpr int kLwASub = kLwM * kLwKSub * 2;      // 16 KB
constexpr int kLwBSub = kLwBRows * kLwKSub * 2;  // 16 KB
constexpr int kLwABytes = kLwSubs * kLwASub;
constexpr int kLwBBytes = kLwSubs * kLwBSub;
constexpr int kLwStageBytes = kLwABytes + kLwBBytes;
constexpr int kLwStages = 3;
constexpr uint32_t kLwTmemCols = 2 * kLwN;
constexpr int kLwYBufBytes = 32 * (kLwN / 2) * 2;  // one epilogue warp: 32 rows x 128 bf16
constexpr int kLwSmem = 1024 /* alignment slack */ + kLwStages * kLwStageBytes + 4 * kLwYBufBytes +
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
    int64_t num_m;  // token tiles
    int num_n;      // channel tiles
    int nk;     // k-steps per tile
};

// Tile order: groups of kLwGroupM token blocks; inside a group the channel
// block varies slowest, so the ~74 tiles in flight share a few Wo blocks
// (3.7 MB each at k = 7168) and one group of X rows in L2, and Wo is read from
// DRAM once per group instead of once per wave.
constexpr int kLwGroupM = 8;

__device__ __forceinline__ void tile_coords(int64_t tile, int64_t num_m, int num_n, int32_t &m0,
                                            int32_t &n0) {
    const int64_t group_tiles = (int64_t)kLwGroupM * num_n;
    const int64_t g = tile / group_tiles;
    const int64_t rem = tile - g * group_tiles;
    const int64_t m_base = g * kLwGroupM;
    const int64_t gm = num_m - m_base < kLwGroupM ? num_m - m_base : kLwGroupM;
    m0 = (int32_t)((m_base + rem % gm) * kLwTileM);
    n0 = (int32_t)((rem / gm) * kLwN);
}

__device__ __forceinline__ void store_bf16x8_cs(__nv_bfloat16 *p, const float (&v)[8]) {
    uint4 q;
    q.x = pack_bf16x2_rn(v[0], v[1]);
    q.y = pack_bf16x2_rn(v[2], v[3]);
    q.z = pack_bf16x2_rn(v[4], v[5]);
    q.w = pack_bf16x2_rn(v[6], v[7]);
    __stcs(reinterpret_cast<uint4 *>(p), q);
}

template <int N>
__global__ void __launch_bounds__(kLwThreads, 1)
hc_linear_write_kernel(const __grid_constant__ CUtensorMap mapX,
                       const __grid_constant__ CUtensorMap mapW, LinearWriteParams p, int *fault) {
    extern __shared__ __align__(1024) unsigned char smem_raw[];
    unsigned char *smem = reinterpret_cast<unsigned char *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    constexpr int S = kLwStages;
    uint64_t *full = reinterpret_cast<uint64_t *>(smem + S * kLwStageBytes + 4 * kLwYBufBytes);
    uint64_t *empty = full + S;
    uint64_t *acc_full = empty + S;      // [2]
    uint64_t *acc_empty = acc_full + 2;  // [2]
    uint64_t *drained = acc_empty + 2;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(drained + 1);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_slot + 1);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const uint32_t rank = cluster_ctarank();  // 0: the leader, which issues the MMAs
    const bool leader = rank == 0;
    const int64_t pair = blockIdx.x >> 1;
    const int64_t npairs = gridDim.x >> 1;

    if (threadIdx.x == 0) {
        for (int s = 0; s < S; ++s) {
            mbar_init(&full[s], 1);   // leader: its producer's expect_tx (+ both CTAs' bytes)
            mbar_init(&empty[s], 1);  // the MMA commit, multicast to both CTAs
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(&acc_full[b], 1);   // the MMA commit, multicast to both CTAs
            mbar_init(&acc_empty[b], 8);  // leader: the four epilogue warps of each CTA
        }
        mbar_init(drained, 1);
        *abort_flag = 0;
        fence_barrier_init();
        prefetch_tensor_map(&mapX);
        prefetch_tensor_map(&mapW);
    }
    if (warp == 1) {
        tmem_alloc_pair(tmem_slot, kLwTmemCols);
        tmem_relinquish_pair();
    }
    tc_fence_before_sync();
    cluster_sync_all();  // both CTAs' barriers initialised, TMEM allocated
    tc_fence_after_sync();
    const uint32_t tmem = *tmem_slot;

    if (warp == 0) {
        // ---------------- TMA producer (both CTAs) ----------------
        if (lane == 0) {
            const uint32_t full_leader = mapa_shared(smem_addr(&full[0]), 0);
            int s = 0;
            uint32_t ph = 0;
            int64_t it = 0;
            bool ok = true;
            for (int64_t tile = pair; ok && tile < p.tiles; tile += npairs) {
                int32_t m0, n0;
                tile_coords(tile, p.num_m, p.num_n, m0, n0);
                for (int ks = 0; ks < p.nk; ++ks, ++it) {
                    if (it >= S &&
                        !mbar_wait_bounded(&empty[s], ph ^ 1u, abort_flag, fault, FAULT_WAIT_EMPTY)) {
                        ok = false;
                        break;
                    }
                    unsigned char *st = smem + s * kLwStageBytes;
                    if (leader) mbar_arrive_expect_tx(&full[s], (uint32_t)(2 * kLwStageBytes));
#pragma unroll
                    for (int c = 0; c < kLwSubs; ++c) {
                        tma_load_2d_pair(st + c * kLwASub, &mapX, ks * kLwK + c * kLwKSub,
                                         m0 + (int32_t)rank * kLwM, full_leader + 8u * (uint32_t)s);
                        tma_load_2d_pair(st + kLwABytes + c * kLwBSub, &mapW, ks * kLwK + c * kLwKSub,
                                         n0 + (int32_t)rank * kLwBRows, full_leader + 8u * (uint32_t)s);
                    }
                    if (++s == S) {
                        s = 0;
                        ph ^= 1u;
                    }
                }
            }
            // the copies still in flight (both CTAs' bytes complete on the
            // leader's barriers) land before the pair leaves
            if (leader)
                for (int64_t q = (it > S ? it - S : 0); q < it; ++q)
                    mbar_wait_drain(&full[q % S], (uint32_t)((q / S) & 1), fault);
        }
        __syncwarp();
    } else if (warp == 1) {
        // ---------------- MMA issuer (the leader) ----------------
        if (lane == 0 && leader) {
            const uint32_t idesc = umma_idesc_bf16_f32(kLwTileM, kLwN);
            int s = 0;
            uint32_t ph = 0;
            int lt = 0;
            bool ok = true;
            for (int64_t tile = pair; ok && tile < p.tiles; tile += npairs, ++lt) {
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
                    for (int c = 0; c < kLwSubs; ++c) {
#pragma unroll
                        for (int kk = 0; kk < kLwKSub / 16; ++kk) {
                            // +32 bytes along K per 16-element step inside the swizzle atom
                            umma_bf16_pair(dacc, umma_desc_sw128(a0 + c * kLwASub + kk * 32),
                                           umma_desc_sw128(b0 + c * kLwBSub + kk * 32), idesc,
                                           (ks | c | kk) != 0);
                        }
                    }
                    umma_commit_pair(&empty[s], 0x3);  // both CTAs' stages are free once read
                    if (++s == S) {
                        s = 0;
                        ph ^= 1u;
                    }
                }
                if (!ok) break;
                umma_commit_pair(&acc_full[buf], 0x3);  // both halves of the accumulator complete
            }
            umma_commit_pair(drained, 0x1);  // every MMA issued so far has finished
            mbar_wait_drain(drained, 0, fault);
        }
        __syncwarp();
    } else {
        // Warp q owns TMEM lanes (token rows) 32q..32q+31. Per half tile (128
        // channels): (A) each thread loads its row's 128 accumulators, rounds
        // them to bf16 and parks them in the warp's 8 KB slice of shared
        // memory (16-byte chunks XOR-swizzled by row, so neither the row-wise
        // writes nor the column-wise reads conflict); (B) the warp then walks
        // its rows two at a time, a half-warp per row, each lane taking 8
        // channels: the stream loads and H' stores are 256-byte coalesced
        // runs. The accumulator is released right after the last TMEM load.
        const int quarter = warp & 3;  // TMEM lanes this warp may access
        const uint32_t lane_base = tmem + ((uint32_t)(quarter * 32) << 16);
        unsigned char *ybuf = smem + S * kLwStageBytes + quarter * kLwYBufBytes;
        // row pairs per iteration: as many as the registers hold (packed bf16)
        constexpr int RPI = N <= 1 ? 16 : N <= 2 ? 8 : N <= 4 ? 4 : 1;
        const int half_lane = lane >> 4;  // which row of the pair
        const int lc = lane & 15;         // 16-byte chunk of the row (8 channels)
        int lt = 0;
        const uint32_t acc_empty_leader = mapa_shared(smem_addr(&acc_empty[0]), 0);
        for (int64_t tile = pair; tile < p.tiles; tile += npairs, ++lt) {
            const int buf = lt & 1;
            const bool w = mbar_wait_bounded(&acc_full[buf], (uint32_t)((lt >> 1) & 1), abort_flag,
                                             fault, FAULT_WAIT_FULL);
            if (!__all_sync(0xffffffffu, w)) break;
            tc_fence_after_sync();
            int32_t m0, n0;
            tile_coords(tile, p.num_m, p.num_n, m0, n0);
            const int64_t t0 = (int64_t)m0 + (int64_t)rank * kLwM + quarter * 32;  // this warp's first row
#pragma unroll 1
            for (int hf = 0; hf < 2; ++hf) {
                // (A) accumulators -> bf16 -> shared memory (row = lane)
#pragma unroll
                for (int c0 = 0; c0 < kLwN / 2; c0 += 16) {
                    uint32_t v[16];
                    tmem_ld_32x32b_x16(lane_base + (uint32_t)(buf * kLwN + hf * (kLwN / 2) + c0), v);
                    tmem_ld_wait();
                    uint4 q0, q1;
                    q0.x = pack_bf16x2_rn(__uint_as_float(v[0]), __uint_as_float(v[1]));
                    q0.y = pack_bf16x2_rn(__uint_as_float(v[2]), __uint_as_float(v[3]));
                    q0.z = pack_bf16x2_rn(__uint_as_float(v[4]), __uint_as_float(v[5]));
                    q0.w = pack_bf16x2_rn(__uint_as_float(v[6]), __uint_as_float(v[7]));
                    q1.x = pack_bf16x2_rn(__uint_as_float(v[8]), __uint_as_float(v[9]));
                    q1.y = pack_bf16x2_rn(__uint_as_float(v[10]), __uint_as_float(v[11]));
                    q1.z = pack_bf16x2_rn(__uint_as_float(v[12]), __uint_as_float(v[13]));
                    q1.w = pack_bf16x2_rn(__uint_as_float(v[14]), __uint_as_float(v[15]));
                    const int ch = c0 >> 3;  // logical chunk (even)
                    *reinterpret_cast<uint4 *>(ybuf + lane * 256 + ((ch ^ (lane & 7)) << 4)) = q0;
                    *reinterpret_cast<uint4 *>(ybuf + lane * 256 + (((ch + 1) ^ (lane & 7)) << 4)) = q1;
                }
                if (hf == 1) {
                    // every accumulator of this tile is in registers or shared memory
                    tc_fence_before_sync();
                    __syncwarp();
                    if (lane == 0) mbar_arrive_cluster(acc_empty_leader + 8u * (uint32_t)buf);
                }
                __syncwarp();
                // (B) rows in pairs, coalesced along the channels. The stream
                // slices of RPI row pairs are loaded (packed bf16) before any
                // is mixed, so each iteration keeps RPI * n * 512 bytes per
                // warp in flight.
                const int64_t c = n0 + hf * (kLwN / 2) + lc * 8;
                for (int rr = 0; rr < 32; rr += 2 * RPI) {
                    uint4 hraw[RPI][N], yraw[RPI];
                    bool live[RPI];
                    int64_t t[RPI];
#pragma unroll
                    for (int u = 0; u < RPI; ++u) {
                        const int row = rr + 2 * u + half_lane;
                        t[u] = t0 + row;
                        live[u] = t[u] < p.T && c < p.d;
                        yraw[u] = *reinterpret_cast<const uint4 *>(ybuf + row * 256 + ((lc ^ (row & 7)) << 4));
                        if (live[u]) {
                            const __nv_bfloat16 *Ht = p.H + t[u] * N * p.d + c;
#pragma unroll
                            for (int i = 0; i < N; ++i)
                                hraw[u][i] = __ldcs(reinterpret_cast<const uint4 *>(Ht + i * p.d));
                        }
                    }
#pragma unroll
                    for (int u = 0; u < RPI; ++u) {
                        if (!live[u]) continue;
                        if (p.y) *reinterpret_cast<uint4 *>(p.y + t[u] * p.d + c) = yraw[u];
                        float hv[N][8], yv[8];
#pragma unroll
                        for (int i = 0; i < N; ++i) {
                            widen_bf16x2(hraw[u][i].x, hv[i][0], hv[i][1]);
                            widen_bf16x2(hraw[u][i].y, hv[i][2], hv[i][3]);
                            widen_bf16x2(hraw[u][i].z, hv[i][4], hv[i][5]);
                            widen_bf16x2(hraw[u][i].w, hv[i][6], hv[i][7]);
                        }
                        widen_bf16x2(yraw[u].x, yv[0], yv[1]);
                        widen_bf16x2(yraw[u].y, yv[2], yv[3]);
                        widen_bf16x2(yraw[u].z, yv[4], yv[5]);
                        widen_bf16x2(yraw[u].w, yv[6], yv[7]);
                        // the row's parameters (stride 0: shared by all tokens), L1 broadcasts
                        const float *Ap = p.A + t[u] * p.A_s;
                        const float *bp = p.b + t[u] * p.b_s;
                        __nv_bfloat16 *Hot = p.Hout + t[u] * N * p.d + c;
#pragma unroll
                        for (int j = 0; j < N; ++j) {
                            float acc[8];
#pragma unroll
                            for (int e = 0; e < 8; ++e) acc[e] = -0.0f;
#pragma unroll
                            for (int i = 0; i < N; ++i) {
                                const float aij = Ap[i * N + j];
#pragma unroll
                                for (int e = 0; e < 8; ++e) acc[e] = __fmaf_rn(aij, hv[i][e], acc[e]);
                            }
                            const float bj = bp[j];
#pragma unroll
                            for (int e = 0; e < 8; ++e) acc[e] = __fmaf_rn(bj, yv[e], acc[e]);
                            store_bf16x8_cs(Hot + j * p.d, acc);
                        }
                    }
                }
                __syncwarp();  // the slice is rewritten by the next half / tile
            }
        }
    }

    // every role of both CTAs has finished with TMEM and with the peer's
    // shared memory (the leader drained its MMAs and the pair's copies)
    tc_fence_before_sync();
    cluster_sync_all();
    if (warp == 1) {
        tc_fence_after_sync();
        tmem_dealloc_pair(tmem, kLwTmemCols);
    }
}

template <int N>
hc_status launch_n_lw(const CUtensorMap &mapX, const CUtensorMap &mapW, const LinearWriteParams &lp,
                      const LaunchCtx &ctx, cudaStream_t st) {
    auto kern = hc_linear_write_kernel<N>;
    static std::atomic<bool> configured[64];
    if (ctx.device < 0 || ctx.device >= 64)
        return set_error(HC_ERR_UNSUPPORTED, "device ordinal %d >= 64", ctx.device);
    if (!configured[ctx.device].load()) {
        cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, kLwSmem);
        if (e != cudaSuccess)
            return set_error(HC_ERR_CUDA, "cudaFuncSetAttribute(%d B smem): %s", kLwSmem,
                             cudaGetErrorString(e));
        configured[ctx.device].store(true);
    }
    // one CTA pair (a cluster of two) per two SMs, at most one pair per tile
    int64_t pairs = ctx.sms / 2;
    if (pairs > lp.tiles) pairs = lp.tiles;
    if (pairs < 1) pairs = 1;
    cudaLaunchConfig_t cfg{};
    cfg.gridDim = dim3((unsigned)(2 * pairs), 1, 1);
    cfg.blockDim = dim3(kLwThreads, 1, 1);
    cfg.dynamicSmemBytes = kLwSmem;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 2;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    cudaError_t e = cudaLaunchKernelEx(&cfg, kern, mapX, mapW, lp, ctx.fault);
    if (e == cudaSuccess) e = cudaGetLastError();
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
    const int64_t num_m = (a.T + kLwTileM - 1) / kLwTileM;
    const int64_t num_n = (a.d + kLwN - 1) / kLwN;
    const int64_t nk = (a.k + kLwK - 1) / kLwK;
    if (num_m > (int64_t(1) << 31) / kLwTileM || num_n > INT32_MAX / kLwN || nk > INT32_MAX / kLwK)
        return set_error(HC_ERR_UNSUPPORTED, "shape too large for the tile grid");
    lp.num_n = (int)num_n;
    lp.num_m = num_m;
    lp.tiles = num_m * num_n;
    lp.nk = (int)nk;

    CUtensorMap mapX, mapW;
    hc_status ms = make_tma_map_bf16(&mapX, a.X, (uint64_t)a.k, (uint64_t)a.T, kLwKSub, kLwM);
    if (ms != HC_OK) return ms;
    ms = make_tma_map_bf16(&mapW, a.Wo, (uint64_t)a.k, (uint64_t)a.d, kLwKSub, kLwBRows);
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
