// hc_logits.cu -- input-dependent mixing logits on the tensor cores.
//
//   z[t][j] = r_t * sum_k u_t[k] * W[j][k],   u_t = H[t] flattened (n*d),
//   r_t = 1 / sqrt(sum_k u_t[k]^2 / (n*d) + eps)
//
// a GEMM [T x nd] x [nd x P] with a per-row RMS scale. Each CTA owns a tile of
// `rows` tokens (<= 128; chosen so every SM gets one tile) and the whole K:
//   warp 0      TMA producer: per k-step of 256, four adjacent 128B-swizzled
//               sub-tiles of H (rows x 64) and of W (Npad x 64), so each
//               token row is fetched 512 contiguous bytes at a time, into a
//               ring of shared-memory stages;
//   warp 1      allocates TMEM; one lane issues tcgen05.mma (M = 128, N = Npad,
//               K = 16 per instruction, bf16 x bf16 -> fp32 in TMEM) and
//               commits each stage back to the producer;
//   warps 2-5   read each H tile for the fp64 sum of squares of their row
//               (one thread per TMEM lane), then load the accumulator from
//               TMEM, scale by r_t and store z.
// Every wait is bounded; on time-out the CTA records a fault, drains its
// copies and MMAs, frees TMEM and exits.
#include <cuda.h>
#include <cudaTypedefs.h>

#include <atomic>

#include "hc_launch.h"
#include "hc_tc.cuh"

namespace hc {

namespace {

constexpr int kLgThreads = 192;
constexpr int kLgKSub = 64;   // bf16 elements per sub-tile (one 128-byte swizzle row)
constexpr int kLgSubs = 4;    // sub-tiles per stage: 512 contiguous bytes of each row
constexpr int kLgKStep = kLgKSub * kLgSubs;
constexpr int kLgM = 128;     // MMA rows (TMEM lanes)
constexpr int kLgMaxStages = 6;

struct LogitsParams {
    float *z;
    int64_t T;
    int64_t K;       // n * d
    int P;           // logits per token
    int Npad;        // P rounded up to 16 (MMA N)
    int rows;        // tokens per CTA tile (<= 128, multiple of 8)
    int a_bytes;     // A region of a stage: kLgSubs sub-tiles of rows x 128 B + MMA read pad
    int nk;          // k-steps
    int stages;
    uint32_t tmem_cols;
    float eps;
};

__global__ void __launch_bounds__(kLgThreads, 1)
hc_logits_kernel(const __grid_constant__ CUtensorMap mapH, const __grid_constant__ CUtensorMap mapW,
                 LogitsParams p, int *fault) {
    extern __shared__ __align__(1024) unsigned char smem_raw[];
    // 1024-byte aligned base for the swizzle atoms
    unsigned char *smem = reinterpret_cast<unsigned char *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const int a_bytes = p.a_bytes;
    const int a_sub = p.rows * 128;   // bytes of one A sub-tile (1024-aligned: rows % 8 == 0)
    const int b_sub = p.Npad * 128;
    const int stage_bytes = a_bytes + kLgSubs * b_sub;
    uint64_t *full = reinterpret_cast<uint64_t *>(smem + (size_t)p.stages * stage_bytes);
    uint64_t *empty = full + p.stages;
    uint64_t *accum = empty + p.stages;
    uint64_t *done = accum + 1;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(done + 1);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_slot + 1);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int S = p.stages;

    if (threadIdx.x == 0) {
        for (int s = 0; s < S; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1 + 4);  // the MMA commit + the four statistic warps
        }
        mbar_init(accum, 1);
        mbar_init(done, 4);
        *abort_flag = 0;
        fence_barrier_init();
        prefetch_tensor_map(&mapH);
        prefetch_tensor_map(&mapW);
    }
    if (warp == 1) {
        tmem_alloc(tmem_slot, p.tmem_cols);
        tmem_relinquish();
    }
    tc_fence_before_sync();
    __syncthreads();
    tc_fence_after_sync();
    const uint32_t tmem_d = *tmem_slot;
    const int64_t row0 = (int64_t)blockIdx.x * p.rows;

    if (warp == 0) {
        // ---------------- producer ----------------
        if (lane == 0) {
            const uint32_t tx = (uint32_t)(kLgSubs * (a_sub + b_sub));
            int s = 0;
            uint32_t ph = 0;
            int ks = 0;
            for (; ks < p.nk; ++ks) {
                if (ks >= S && !mbar_wait_bounded(&empty[s], ph ^ 1u, abort_flag, fault, FAULT_WAIT_EMPTY))
                    break;
                unsigned char *st = smem + (size_t)s * stage_bytes;
                mbar_arrive_expect_tx(&full[s], tx);
#pragma unroll
                for (int c = 0; c < kLgSubs; ++c)
                    tma_load_2d(st + c * a_sub, &mapH, ks * kLgKStep + c * kLgKSub, (int32_t)row0, &full[s]);
#pragma unroll
                for (int c = 0; c < kLgSubs; ++c)
                    tma_load_2d(st + a_bytes + c * b_sub, &mapW, ks * kLgKStep + c * kLgKSub, 0, &full[s]);
                if (++s == S) {
                    s = 0;
                    ph ^= 1u;
                }
            }
            for (int q = (ks > S ? ks - S : 0); q < ks; ++q)
                mbar_wait_drain(&full[q % S], (uint32_t)((q / S) & 1), fault);
        }
        return;
    }

    if (warp == 1) {
        // ---------------- MMA issuer ----------------
        if (lane == 0) {
            const uint32_t idesc = umma_idesc_bf16_f32(kLgM, p.Npad);
            int s = 0;
            uint32_t ph = 0;
            for (int ks = 0; ks < p.nk; ++ks) {
                if (!mbar_wait_bounded(&full[s], ph, abort_flag, fault, FAULT_WAIT_FULL)) break;
                tc_fence_after_sync();
                const uint32_t a0 = smem_addr(smem + (size_t)s * stage_bytes);
                const uint32_t b0 = a0 + (uint32_t)a_bytes;
#pragma unroll
                for (int c = 0; c < kLgSubs; ++c) {
#pragma unroll
                    for (int kk = 0; kk < kLgKSub / 16; ++kk) {
                        // +32 bytes along K per 16-element MMA step inside the swizzle atom
                        umma_bf16(tmem_d, umma_desc_sw128(a0 + c * a_sub + kk * 32),
                                  umma_desc_sw128(b0 + c * b_sub + kk * 32), idesc,
                                  (ks | c | kk) != 0);
                    }
                }
                umma_commit(&empty[s]);  // stage free once these MMAs have read it
                if (++s == S) {
                    s = 0;
                    ph ^= 1u;
                }
            }
            umma_commit(accum);  // accumulator complete (or, after a time-out, quiet)
            mbar_wait_drain(accum, 0, fault);
        }
        __syncwarp();
        // the epilogue warps are done with TMEM before it is freed
        mbar_wait_drain(done, 0, fault);
        tc_fence_after_sync();
        tmem_dealloc(tmem_d, p.tmem_cols);
        return;
    }

    // ---------------- statistic + epilogue (warps 2..5) ----------------
    const int quarter = warp & 3;  // TMEM lanes this warp may access
    const int r = quarter * 32 + lane;  // tile row = TMEM lane
    const int64_t t = row0 + r;
    const bool live = r < p.rows && t < p.T;
    double ss = 0.0;
    bool ok = true;
    {
        int s = 0;
        uint32_t ph = 0;
        for (int ks = 0; ks < p.nk; ++ks) {
            const bool w = mbar_wait_bounded(&full[s], ph, abort_flag, fault, FAULT_WAIT_FULL);
            if (!__all_sync(0xffffffffu, w)) {
                ok = false;
                break;
            }
            if (live) {
                // In each sub-tile the row's 128 bytes (64 bf16) fill one
                // 128-byte line, its 16-byte chunks permuted by the swizzle;
                // the sum takes them in any order. Starting each row at
                // physical chunk (row & 7) keeps the eight rows a quarter-warp
                // reads on distinct banks.
                const unsigned char *rowp = smem + (size_t)s * stage_bytes + (size_t)r * 128;
                const int rot = r & 7;
                float2 acc0 = make_float2(0.0f, 0.0f), acc1 = make_float2(0.0f, 0.0f);
#pragma unroll
                for (int c = 0; c < 8 * kLgSubs; ++c) {
                    const uint4 q = *reinterpret_cast<const uint4 *>(
                        rowp + (size_t)(c >> 3) * a_sub + (size_t)(((c & 7) ^ rot) * 16));
                    float2 v;
                    widen_bf16x2(q.x, v.x, v.y);
                    acc0 = ffma2_rn(v, v, acc0);
                    widen_bf16x2(q.y, v.x, v.y);
                    acc1 = ffma2_rn(v, v, acc1);
                    widen_bf16x2(q.z, v.x, v.y);
                    acc0 = ffma2_rn(v, v, acc0);
                    widen_bf16x2(q.w, v.x, v.y);
                    acc1 = ffma2_rn(v, v, acc1);
                }
                ss += ((double)acc0.x + (double)acc0.y) + ((double)acc1.x + (double)acc1.y);
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(&empty[s]);
            if (++s == S) {
                s = 0;
                ph ^= 1u;
            }
        }
    }
    if (ok) {
        const bool w = mbar_wait_bounded(accum, 0, abort_flag, fault, FAULT_WAIT_REDUCE);
        ok = __all_sync(0xffffffffu, w);
    }
    if (ok) {
        tc_fence_after_sync();
        const float rs = __double2float_rn(1.0 / sqrt(ss / (double)p.K + (double)p.eps));
        float *zt = p.z + t * p.P;
        for (int c0 = 0; c0 < p.Npad; c0 += 16) {
            uint32_t v[16];
            tmem_ld_32x32b_x16(tmem_d + ((uint32_t)(quarter * 32) << 16) + (uint32_t)c0, v);
            tmem_ld_wait();
            if (live) {
#pragma unroll
                for (int j = 0; j < 16; ++j)
                    if (c0 + j < p.P) zt[c0 + j] = __fmul_rn(__uint_as_float(v[j]), rs);
            }
        }
    }
    tc_fence_before_sync();
    __syncwarp();
    if (lane == 0) mbar_arrive(done);
}

}  // namespace

// 2-D bf16 tensor map with 128-byte swizzle and zero fill out of bounds.
// cuTensorMapEncodeTiled through the runtime's driver entry point (the library
// does not link the driver library directly).
static PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
    // looked up once (thread-safe static initialisation); null if unavailable
    static const PFN_cuTensorMapEncodeTiled_v12000 fn = [] {
        void *ptr = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) !=
                cudaSuccess ||
            q != cudaDriverEntryPointSuccess)
            ptr = nullptr;
        return reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(ptr);
    }();
    return fn;
}

hc_status make_tma_map_bf16(CUtensorMap *map, const void *base, uint64_t inner, uint64_t outer,
                            uint32_t box_inner, uint32_t box_outer) {
    auto fn = encode_fn();
    if (!fn) return set_error(HC_ERR_CUDA, "cuTensorMapEncodeTiled is not available");
    cuuint64_t gdim[2] = {inner, outer};
    cuuint64_t gstride[1] = {inner * 2};
    cuuint32_t box[2] = {box_inner, box_outer};
    cuuint32_t estride[2] = {1, 1};
    CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void *>(base), gdim, gstride,
                    box, estride, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                    CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) return set_error(HC_ERR_CUDA, "cuTensorMapEncodeTiled failed (%d)", (int)r);
    return HC_OK;
}

hc_status launch_mix_logits(const void *H, const void *W, float *z, int64_t T, int n, int64_t d,
                            int P, float eps, const LaunchCtx &ctx, cudaStream_t st) {
    LogitsParams lp{};
    lp.z = z;
    lp.T = T;
    lp.K = (int64_t)n * d;
    lp.P = P;
    lp.Npad = (P + 15) / 16 * 16;
    lp.eps = eps;
    // tokens per tile: spread T over the SMs, a multiple of 8 rows, at most 128
    int64_t rows = (T + ctx.sms - 1) / ctx.sms;
    rows = (rows + 7) / 8 * 8;
    if (rows > kLgM) rows = kLgM;
    if (rows < 8) rows = 8;
    lp.rows = (int)rows;
    const int64_t nk = (lp.K + kLgKStep - 1) / kLgKStep;
    if (nk > INT32_MAX) return set_error(HC_ERR_UNSUPPORTED, "n*d too large");
    lp.nk = (int)nk;
    uint32_t cols = 32;
    while (cols < (uint32_t)lp.Npad) cols <<= 1;
    lp.tmem_cols = cols;
    // the M = 128 MMA reads 128 rows from each sub-tile base: pad the A region
    // so the last sub-tile's read stays inside the stage (rows beyond `rows`
    // feed TMEM lanes the epilogue ignores)
    lp.a_bytes = kLgSubs * lp.rows * 128 + (kLgM - lp.rows) * 128;
    const int stage_bytes = lp.a_bytes + kLgSubs * lp.Npad * 128;
    const int fixed = 1024 /* alignment slack */ + 2 * kLgMaxStages * 8 + 16 + 16;
    int stages = (kSmemLimitLogits - fixed) / stage_bytes;
    if (stages > kLgMaxStages) stages = kLgMaxStages;
    if (stages < 2) return set_error(HC_ERR_UNSUPPORTED, "P = %d leaves no room for two stages", P);
    lp.stages = stages;
    const int smem = fixed + stages * stage_bytes;

    CUtensorMap mapH, mapW;
    hc_status ms = make_tma_map_bf16(&mapH, H, (uint64_t)lp.K, (uint64_t)T, kLgKSub, (uint32_t)lp.rows);
    if (ms != HC_OK) return ms;
    ms = make_tma_map_bf16(&mapW, W, (uint64_t)lp.K, (uint64_t)P, kLgKSub, (uint32_t)lp.Npad);
    if (ms != HC_OK) return ms;

    static std::atomic<int> configured[64];  // largest dynamic smem opted in so far, per device
    if (ctx.device < 0 || ctx.device >= 64)
        return set_error(HC_ERR_UNSUPPORTED, "device ordinal %d >= 64", ctx.device);
    if (smem > configured[ctx.device].load()) {
        cudaError_t e = cudaFuncSetAttribute(hc_logits_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             smem);
        if (e != cudaSuccess)
            return set_error(HC_ERR_CUDA, "cudaFuncSetAttribute(%d B smem): %s", smem,
                             cudaGetErrorString(e));
        configured[ctx.device].store(smem);
    }
    const int64_t grid = (T + lp.rows - 1) / lp.rows;
    hc_logits_kernel<<<(unsigned)grid, kLgThreads, smem, st>>>(mapH, mapW, lp, ctx.fault);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return set_error(HC_ERR_CUDA, "hc_logits_kernel launch: %s", cudaGetErrorString(e));
    return HC_OK;
}

}  // namespace hc
