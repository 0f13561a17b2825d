// hc_device.cuh -- device helpers for the Hyper-Connections step on sm_100a:
// 16-byte vector I/O of the storage dtype, and the per-token parameter
// preparation (Sinkhorn projection and read-weight softmax) done by small
// lane groups in registers.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace hc {

constexpr int kMaxStreams = 8;
// Largest CTA of the register-streaming kernels; with 8 slices per thread it
// bounds d of a normalising call at 512 * 8 vectors.
constexpr int kStreamMaxThreads = 512;

// Step kinds: read + RMSNorm, write mix, fused write then read.
enum Kind { KIND_READ = 0, KIND_WRITE = 1, KIND_FUSED = 2 };

// ---------------------------------------------------------------------------
// Storage dtype traits: one 16-byte vector = V elements.
// ---------------------------------------------------------------------------
template <typename S> struct StorageTraits;

template <> struct StorageTraits<float> {
    static constexpr int V = 4;
};
template <> struct StorageTraits<__nv_bfloat16> {
    static constexpr int V = 8;
};

// Streaming (evict-first) 16-byte load, widened to fp32 (exact).
__device__ __forceinline__ void load_vec_cs(const float *p, float (&v)[4]) {
    float4 q = __ldcs(reinterpret_cast<const float4 *>(p));
    v[0] = q.x; v[1] = q.y; v[2] = q.z; v[3] = q.w;
}
__device__ __forceinline__ void widen_bf16x2(uint32_t w, float &lo, float &hi) {
    lo = __uint_as_float(w << 16);
    hi = __uint_as_float(w & 0xffff0000u);
}
__device__ __forceinline__ void load_vec_cs(const __nv_bfloat16 *p, float (&v)[8]) {
    uint4 q = __ldcs(reinterpret_cast<const uint4 *>(p));
    widen_bf16x2(q.x, v[0], v[1]);
    widen_bf16x2(q.y, v[2], v[3]);
    widen_bf16x2(q.z, v[4], v[5]);
    widen_bf16x2(q.w, v[6], v[7]);
}

// Round to the storage dtype (RNE), store 16 bytes with the streaming policy,
// and hand back the rounded values as fp32 (what a later read of the stored
// tensor would see).
__device__ __forceinline__ void store_vec_cs(float *p, const float (&v)[4], float (&stored)[4]) {
    __stcs(reinterpret_cast<float4 *>(p), make_float4(v[0], v[1], v[2], v[3]));
#pragma unroll
    for (int e = 0; e < 4; ++e) stored[e] = v[e];
}
__device__ __forceinline__ uint32_t pack_bf16x2_rn(float lo, float hi) {
    __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);  // .x = lo (low half)
    return *reinterpret_cast<uint32_t *>(&h);
}
__device__ __forceinline__ void store_vec_cs(__nv_bfloat16 *p, const float (&v)[8],
                                             float (&stored)[8]) {
    uint4 q;
    q.x = pack_bf16x2_rn(v[0], v[1]);
    q.y = pack_bf16x2_rn(v[2], v[3]);
    q.z = pack_bf16x2_rn(v[4], v[5]);
    q.w = pack_bf16x2_rn(v[6], v[7]);
    __stcs(reinterpret_cast<uint4 *>(p), q);
    widen_bf16x2(q.x, stored[0], stored[1]);
    widen_bf16x2(q.y, stored[2], stored[3]);
    widen_bf16x2(q.z, stored[4], stored[5]);
    widen_bf16x2(q.w, stored[6], stored[7]);
}
__device__ __forceinline__ void store_vec_cs(float *p, const float (&v)[4]) {
    __stcs(reinterpret_cast<float4 *>(p), make_float4(v[0], v[1], v[2], v[3]));
}
__device__ __forceinline__ void store_vec_cs(__nv_bfloat16 *p, const float (&v)[8]) {
    uint4 q;
    q.x = pack_bf16x2_rn(v[0], v[1]);
    q.y = pack_bf16x2_rn(v[2], v[3]);
    q.z = pack_bf16x2_rn(v[4], v[5]);
    q.w = pack_bf16x2_rn(v[6], v[7]);
    __stcs(reinterpret_cast<uint4 *>(p), q);
}

// Read-only (L1-cached) load of V fp32 gains.
template <int V>
__device__ __forceinline__ void load_gain(const float *g, int64_t k, float (&gv)[V]) {
    if (g == nullptr) {
#pragma unroll
        for (int e = 0; e < V; ++e) gv[e] = 1.0f;
        return;
    }
#pragma unroll
    for (int e = 0; e < V; e += 4) {
        float4 q = __ldg(reinterpret_cast<const float4 *>(g + k + e));
        gv[e] = q.x; gv[e + 1] = q.y; gv[e + 2] = q.z; gv[e + 3] = q.w;
    }
}

// ---------------------------------------------------------------------------
// Lane groups for the per-token n x n parameters.
//
// A warp is split into groups of GL lanes; each group owns one token, and
// lane q of a group holds elements e = q + GL * r (r < EPL) of the row-major
// n x n matrix. GL is the power of two >= n*n capped at 32, so n <= 4 packs
// several tokens per warp and n = 6..8 holds two elements per lane.
// ---------------------------------------------------------------------------
template <int N> struct Group {
    static constexpr int NN = N * N;
    static constexpr int GL = NN <= 1 ? 1 : NN <= 2 ? 2 : NN <= 4 ? 4 : NN <= 8 ? 8
                              : NN <= 16 ? 16 : 32;
    static constexpr int EPL = (NN + GL - 1) / GL;
    static constexpr int TPW = 32 / GL;  // tokens per warp
};

// Value of element `ep` of this lane's group (all 32 lanes must call).
template <int N>
__device__ __forceinline__ float group_fetch(const float (&m)[Group<N>::EPL], int base, int ep) {
    constexpr int GL = Group<N>::GL;
    const int src = base + (ep & (GL - 1));
    float v0 = __shfl_sync(0xffffffffu, m[0], src);
    if constexpr (Group<N>::EPL == 1) {
        return v0;
    } else {
        float v1 = __shfl_sync(0xffffffffu, m[1], src);
        return (ep >= GL) ? v1 : v0;
    }
}

// Sinkhorn projection of the group's matrix, in place: m = exp(L) on entry
// is NOT assumed; the caller passes the logits and this computes
//   M = exp(L); K times { rows /= row sums; columns /= column sums }.
// Sums run in index order starting from +0, divisions are IEEE (__fdiv_rn),
// so the operation sequence per element is fixed. All lanes of the warp call
// this with the same K.
template <int N>
__device__ __forceinline__ void group_sinkhorn(float (&m)[Group<N>::EPL], int lane, int K) {
    constexpr int NN = N * N, GL = Group<N>::GL, EPL = Group<N>::EPL;
    const int q = lane & (GL - 1);
    const int base = lane & ~(GL - 1);
#pragma unroll
    for (int r = 0; r < EPL; ++r) m[r] = expf(m[r]);
    int row[EPL], col[EPL];
#pragma unroll
    for (int r = 0; r < EPL; ++r) {
        int e = q + GL * r;
        e = e < NN ? e : NN - 1;  // idle lanes shadow the last element
        row[r] = e / N;
        col[r] = e - (e / N) * N;
    }
    for (int it = 0; it < K; ++it) {
        float s[EPL];
#pragma unroll
        for (int r = 0; r < EPL; ++r) {
            float acc = 0.0f;
#pragma unroll
            for (int jj = 0; jj < N; ++jj) acc = __fadd_rn(acc, group_fetch<N>(m, base, row[r] * N + jj));
            s[r] = acc;
        }
#pragma unroll
        for (int r = 0; r < EPL; ++r) m[r] = __fdiv_rn(m[r], s[r]);
#pragma unroll
        for (int r = 0; r < EPL; ++r) {
            float acc = 0.0f;
#pragma unroll
            for (int ii = 0; ii < N; ++ii) acc = __fadd_rn(acc, group_fetch<N>(m, base, ii * N + col[r]));
            s[r] = acc;
        }
#pragma unroll
        for (int r = 0; r < EPL; ++r) m[r] = __fdiv_rn(m[r], s[r]);
    }
}

// Softmax over the n read logits of the group's token. Lane q < N holds l_q
// on entry and a_q on exit. Max and sum in index order.
template <int N>
__device__ __forceinline__ float group_softmax(float l, int lane) {
    constexpr int GL = Group<N>::GL;
    const int q = lane & (GL - 1);
    const int base = lane & ~(GL - 1);
    float mx = __shfl_sync(0xffffffffu, l, base);
#pragma unroll
    for (int i = 1; i < N; ++i) {
        float v = __shfl_sync(0xffffffffu, l, base + i);
        if (v > mx) mx = v;
    }
    float ex = (q < N) ? expf(__fsub_rn(l, mx)) : 0.0f;
    float s = 0.0f;
#pragma unroll
    for (int i = 0; i < N; ++i) s = __fadd_rn(s, __shfl_sync(0xffffffffu, ex, base + i));
    return __fdiv_rn(ex, s);
}

// ---------------------------------------------------------------------------
// Per-token parameters of one step, as the kernels see them.
// ---------------------------------------------------------------------------
struct StepParams {
    const void *H;
    const void *y;
    void *Hout;
    void *x;
    int64_t T;
    int64_t d;
    const float *A;  // matrix or logits
    int64_t A_s;     // floats between tokens (0 = shared)
    const float *b;
    int64_t b_s;
    const float *a;  // weights or logits
    int64_t a_s;
    const float *g;  // [d] or nullptr
    float eps;
    int K;
    int mix_logits;   // 1: A holds Sinkhorn logits
    int read_logits;  // 1: a holds softmax logits
};

// Fill the shared-memory parameter block for TB tokens of this CTA's token
// sequence (token of slot tt = first + tt * step). Every warp takes TPW
// tokens; lane groups compute Sinkhorn / softmax in registers.
template <int N, bool WRITE, bool READ>
__device__ __forceinline__ void prepare_params(const StepParams &p, int64_t first, int64_t step,
                                               int TB, float *sA, float *sb, float *sa) {
    constexpr int NN = N * N, GL = Group<N>::GL, EPL = Group<N>::EPL, TPW = Group<N>::TPW;
    const int lane = threadIdx.x & 31;
    const int warp = threadIdx.x >> 5;
    const int nwarps = blockDim.x >> 5;
    const int q = lane & (GL - 1);
    for (int slot0 = warp * TPW; slot0 < TB; slot0 += nwarps * TPW) {
        const int tt = slot0 + lane / GL;  // this group's slot
        const int64_t t = first + (int64_t)tt * step;
        const bool live = tt < TB && t < p.T;
        if constexpr (WRITE) {
            float m[EPL];
#pragma unroll
            for (int r = 0; r < EPL; ++r) {
                const int e = q + GL * r;
                m[r] = (live && e < NN) ? p.A[t * p.A_s + e] : 0.0f;
            }
            if (p.mix_logits) group_sinkhorn<N>(m, lane, p.K);  // warp-uniform branch
            if (live) {
#pragma unroll
                for (int r = 0; r < EPL; ++r) {
                    const int e = q + GL * r;
                    if (e < NN) sA[tt * NN + e] = m[r];
                }
                if (q < N) sb[tt * N + q] = p.b[t * p.b_s + q];
            }
        }
        if constexpr (READ) {
            float l = (live && q < N) ? p.a[t * p.a_s + q] : 0.0f;
            if (p.read_logits) l = group_softmax<N>(l, lane);
            if (live && q < N) sa[tt * N + q] = l;
        }
    }
}

}  // namespace hc
