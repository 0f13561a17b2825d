// hc_backward_common.cuh -- pieces shared by the backward kernels of the
// fused HC step (hc_backward.cu): gain loads, storage vectors widened to
// fp32, and the forward recomputation of one slice.
#pragma once

#include "hc_device.cuh"

namespace hc {

// VE fp32 gains (1 when g is null); k is a multiple of VE.
template <int VE>
__device__ __forceinline__ void bw_load_gain(const float *g, int64_t k, float (&gv)[VE]) {
    if (g == nullptr) {
#pragma unroll
        for (int e = 0; e < VE; ++e) gv[e] = 1.0f;
    } else if constexpr (VE == 2) {
        const float2 q = __ldg(reinterpret_cast<const float2 *>(g + k));
        gv[0] = q.x;
        gv[1] = q.y;
    } else {
#pragma unroll
        for (int e = 0; e < VE; e += 4) {
            const float4 q = __ldg(reinterpret_cast<const float4 *>(g + k + e));
            gv[e] = q.x; gv[e + 1] = q.y; gv[e + 2] = q.z; gv[e + 3] = q.w;
        }
    }
}

// VE-element vectors of the storage dtype (16 or 8 bytes), widened to fp32.
template <typename S, int VE> struct BwVec;
template <> struct BwVec<float, 4> {
    static __device__ __forceinline__ void load(const float *p, float (&v)[4]) {
        const float4 q = __ldcs(reinterpret_cast<const float4 *>(p));
        v[0] = q.x; v[1] = q.y; v[2] = q.z; v[3] = q.w;
    }
    static __device__ __forceinline__ void store(float *p, const float (&v)[4]) {
        __stcs(reinterpret_cast<float4 *>(p), make_float4(v[0], v[1], v[2], v[3]));
    }
    static __device__ __forceinline__ void round(float (&)[4]) {}
    static __device__ __forceinline__ void store_smem(float *p, const float (&v)[4]) {
        *reinterpret_cast<float4 *>(p) = make_float4(v[0], v[1], v[2], v[3]);
    }
    static __device__ __forceinline__ void load_smem(const float *p, float (&v)[4]) {
        const float4 q = *reinterpret_cast<const float4 *>(p);
        v[0] = q.x; v[1] = q.y; v[2] = q.z; v[3] = q.w;
    }
};
template <> struct BwVec<float, 2> {
    static __device__ __forceinline__ void load(const float *p, float (&v)[2]) {
        const float2 q = __ldcs(reinterpret_cast<const float2 *>(p));
        v[0] = q.x; v[1] = q.y;
    }
    static __device__ __forceinline__ void store(float *p, const float (&v)[2]) {
        __stcs(reinterpret_cast<float2 *>(p), make_float2(v[0], v[1]));
    }
    static __device__ __forceinline__ void round(float (&)[2]) {}
    static __device__ __forceinline__ void store_smem(float *p, const float (&v)[2]) {
        *reinterpret_cast<float2 *>(p) = make_float2(v[0], v[1]);
    }
    static __device__ __forceinline__ void load_smem(const float *p, float (&v)[2]) {
        const float2 q = *reinterpret_cast<const float2 *>(p);
        v[0] = q.x; v[1] = q.y;
    }
};
template <> struct BwVec<__nv_bfloat16, 4> {
    static __device__ __forceinline__ void load(const __nv_bfloat16 *p, float (&v)[4]) {
        const uint2 q = __ldcs(reinterpret_cast<const uint2 *>(p));
        widen_bf16x2(q.x, v[0], v[1]); widen_bf16x2(q.y, v[2], v[3]);
    }
    static __device__ __forceinline__ void store(__nv_bfloat16 *p, const float (&v)[4]) {
        uint2 q;
        q.x = pack_bf16x2_rn(v[0], v[1]); q.y = pack_bf16x2_rn(v[2], v[3]);
        __stcs(reinterpret_cast<uint2 *>(p), q);
    }
    static __device__ __forceinline__ void round(float (&v)[4]) {
#pragma unroll
        for (int e = 0; e < 4; e += 2) widen_bf16x2(pack_bf16x2_rn(v[e], v[e + 1]), v[e], v[e + 1]);
    }
    // shared-memory copies of values already rounded to bf16 (exact)
    static __device__ __forceinline__ void store_smem(__nv_bfloat16 *p, const float (&v)[4]) {
        uint2 q;
        q.x = pack_bf16x2_rn(v[0], v[1]); q.y = pack_bf16x2_rn(v[2], v[3]);
        *reinterpret_cast<uint2 *>(p) = q;
    }
    static __device__ __forceinline__ void load_smem(const __nv_bfloat16 *p, float (&v)[4]) {
        const uint2 q = *reinterpret_cast<const uint2 *>(p);
        widen_bf16x2(q.x, v[0], v[1]); widen_bf16x2(q.y, v[2], v[3]);
    }
};

// 8-byte vectors for bf16 (16 bytes would double the per-slice registers and
// halve the CTAs per SM); 16-byte fp32 vectors up to n = 4.
template <typename S> constexpr int bw_vec_elems(int n) {
    return sizeof(S) == 2 ? 4 : (n <= 4 ? 4 : 2);
}

struct BwKernelParams {
    StepParams f;
    const void *dHout;
    const void *dx;
    void *dH;
    void *dy;
    float *gA, *gb, *ga;  // per-token sums (gradients w.r.t. the matrix / weights)
    float *dg_part;       // [gridDim.x][d] or null
};

// The forward of one VE-slice from its widened H and y values: H' as stored
// (hs) and h, exactly as the forward kernels compute them (fp32 FMA chains in
// stream order, storage rounding of H').
template <int N, typename S, int VE>
__device__ __forceinline__ void bw_forward_from(const float (&hv)[N][VE], const float (&yv)[VE],
                                                const float *At, const float *bt, const float *at,
                                                float (&hs)[N][VE], float (&h)[VE]) {
    using V = BwVec<S, VE>;
    // paired fp32 FMAs: each element's chain is the scalar one, bit for bit
#pragma unroll
    for (int e = 0; e < VE; ++e) h[e] = -0.0f;
#pragma unroll
    for (int j = 0; j < N; ++j) {
#pragma unroll
        for (int e = 0; e < VE; e += 2) {
            float2 acc = make_float2(-0.0f, -0.0f);
#pragma unroll
            for (int i = 0; i < N; ++i)
                acc = ffma2_rn(make_float2(At[i * N + j], At[i * N + j]),
                               make_float2(hv[i][e], hv[i][e + 1]), acc);
            acc = ffma2_rn(make_float2(bt[j], bt[j]), make_float2(yv[e], yv[e + 1]), acc);
            hs[j][e] = acc.x;
            hs[j][e + 1] = acc.y;
        }
        V::round(hs[j]);
#pragma unroll
        for (int e = 0; e < VE; e += 2) {
            const float2 hh = ffma2_rn(make_float2(at[j], at[j]), make_float2(hs[j][e], hs[j][e + 1]),
                                       make_float2(h[e], h[e + 1]));
            h[e] = hh.x;
            h[e + 1] = hh.y;
        }
    }
}

// The same, loading the slice's H and y rows from global memory first.
template <int N, typename S, int VE>
__device__ __forceinline__ void bw_forward_slice(const S *Ht, const S *Yt, int64_t d, int64_t k,
                                                 const float *At, const float *bt, const float *at,
                                                 float (&hv)[N][VE], float (&yv)[VE],
                                                 float (&hs)[N][VE], float (&h)[VE]) {
    using V = BwVec<S, VE>;
#pragma unroll
    for (int i = 0; i < N; ++i) V::load(Ht + i * d + k, hv[i]);
    V::load(Yt + k, yv);
    bw_forward_from<N, S, VE>(hv, yv, At, bt, at, hs, h);
}

// Per-thread asynchronous copies (cp.async, no registers held while in
// flight) of CB = 8 or 16 bytes to a shared-memory address (32-bit, shared
// window) from global memory; each thread waits on its
// own groups and reads back only what it copied, so no barrier is needed.
template <int CB>
__device__ __forceinline__ void bw_cp_async(unsigned sa, const void *gmem) {
    static_assert(CB == 8 || CB == 16, "chunk of 8 or 16 bytes");
    if constexpr (CB == 16)
        asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(sa), "l"(gmem) : "memory");
    else
        asm volatile("cp.async.ca.shared.global [%0], [%1], 8;" ::"r"(sa), "l"(gmem) : "memory");
}
__device__ __forceinline__ void bw_cp_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int NW>
__device__ __forceinline__ void bw_cp_wait() { asm volatile("cp.async.wait_group %0;" ::"n"(NW) : "memory"); }
__device__ __forceinline__ void bw_cp_wait_all() { asm volatile("cp.async.wait_all;" ::: "memory"); }

// A VE-element storage vector from shared memory, widened to fp32.
template <typename S, int VE>
__device__ __forceinline__ void bw_ld_stage(const unsigned char *p, float (&v)[VE]) {
    if constexpr (sizeof(S) == 2) {
        const uint2 q = *reinterpret_cast<const uint2 *>(p);
        widen_bf16x2(q.x, v[0], v[1]);
        widen_bf16x2(q.y, v[2], v[3]);
    } else if constexpr (VE == 4) {
        const float4 q = *reinterpret_cast<const float4 *>(p);
        v[0] = q.x; v[1] = q.y; v[2] = q.z; v[3] = q.w;
    } else {
        const float2 q = *reinterpret_cast<const float2 *>(p);
        v[0] = q.x; v[1] = q.y;
    }
}

__host__ __device__ constexpr int bw_pow2_ceil(int m) {
    int p = 1;
    while (p < m) p *= 2;
    return p;
}

// Warp sums of M per-lane values in one halving exchange: at each step the
// lanes with the offset's bit set keep the upper half of their values and
// send the lower half, the others the reverse, so P - 1 shuffles (P = M
// rounded up to a power of two, <= 32) replace M butterflies of five. Value m
// ends in lane m * (32 / P) and its copies (the remaining butterfly steps);
// dst[m] is written from there. Summation order: a fixed tree per launch
// shape, so the result is reproducible.
template <int M>
__device__ __forceinline__ void bw_warp_sums_to(const float (&v)[M], float *dst, int lane) {
    static_assert(M <= 32, "at most 32 values per exchange");
    constexpr int P = bw_pow2_ceil(M);
    float w[P];
#pragma unroll
    for (int m = 0; m < P; ++m) w[m] = m < M ? v[m] : 0.0f;
    int o = 16;
#pragma unroll
    for (int h = P / 2; h >= 1; h /= 2) {
        const bool up = (lane & o) != 0;
#pragma unroll
        for (int m = 0; m < h; ++m) {
            const float send = up ? w[m] : w[m + h];
            const float keep = up ? w[m + h] : w[m];
            w[m] = keep + __shfl_xor_sync(0xffffffffu, send, o);
        }
        o >>= 1;
    }
    float s = w[0];
#pragma unroll
    for (; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
    // lane bits 4, 3, ... (one per halving) spell the value index
    constexpr int span = 32 / P;
    const int idx = lane / span;
    if (lane % span == 0 && idx < M) dst[idx] = s;
}

// VE fp32 values to and from shared memory (16- or 8-byte accesses).
template <int VE>
__device__ __forceinline__ void bw_st_f32(float *p, const float (&v)[VE]) {
    if constexpr (VE == 4) *reinterpret_cast<float4 *>(p) = make_float4(v[0], v[1], v[2], v[3]);
    else *reinterpret_cast<float2 *>(p) = make_float2(v[0], v[1]);
}
template <int VE>
__device__ __forceinline__ void bw_ld_f32(const float *p, float (&v)[VE]) {
    if constexpr (VE == 4) {
        const float4 q = *reinterpret_cast<const float4 *>(p);
        v[0] = q.x; v[1] = q.y; v[2] = q.z; v[3] = q.w;
    } else {
        const float2 q = *reinterpret_cast<const float2 *>(p);
        v[0] = q.x; v[1] = q.y;
    }
}

// Stream j of H' as the forward stores it, from the loaded H and y slices.
template <int N, typename S, int VE>
__device__ __forceinline__ void bw_stream_out(const float (&hv)[N][VE], const float (&yv)[VE],
                                              const float *At, const float *bt, int j,
                                              float (&hs)[VE]) {
#pragma unroll
    for (int e = 0; e < VE; ++e) hs[e] = -0.0f;
#pragma unroll
    for (int i = 0; i < N; ++i)
#pragma unroll
        for (int e = 0; e < VE; ++e) hs[e] = __fmaf_rn(At[i * N + j], hv[i][e], hs[e]);
#pragma unroll
    for (int e = 0; e < VE; ++e) hs[e] = __fmaf_rn(bt[j], yv[e], hs[e]);
    BwVec<S, VE>::round(hs);
}

}  // namespace hc
