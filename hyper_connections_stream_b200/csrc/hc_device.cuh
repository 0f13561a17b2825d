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

// Step kinds. READ / WRITE / FUSED are the residual step; the next three are
// the ends of a stack: EXPAND copies one row into the n streams, EXPAND_READ
// also produces layer 0's block input from them, COLLAPSE mixes the n
// streams into one row (no normalisation). REDUCE is FUSED with y the sum of
// R ranks' partial block outputs (the tensor-parallel all-reduce folded into
// the write; pipelined family only).
enum Kind {
    KIND_READ = 0,
    KIND_WRITE = 1,
    KIND_FUSED = 2,
    KIND_EXPAND = 3,
    KIND_EXPAND_READ = 4,
    KIND_COLLAPSE = 5,
    KIND_REDUCE = 6
};

// Kinds that normalise a mixed row (a CTA-wide statistic per token).
__host__ __device__ constexpr bool kind_normalises(int kind) {
    return kind == KIND_READ || kind == KIND_FUSED || kind == KIND_EXPAND_READ || kind == KIND_REDUCE;
}

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

// Paired fp32 arithmetic (sm_100): one instruction performs the operation on
// two independent element pairs, each correctly rounded exactly like the
// scalar __fmaf_rn / __fmul_rn, so results are bit-identical.
__device__ __forceinline__ float2 ffma2_rn(float2 a, float2 b, float2 c) {
    float2 d;
    asm("{\n\t.reg .b64 ra, rb, rc, rd;\n\t"
        "mov.b64 ra, {%2, %3};\n\tmov.b64 rb, {%4, %5};\n\tmov.b64 rc, {%6, %7};\n\t"
        "fma.rn.f32x2 rd, ra, rb, rc;\n\tmov.b64 {%0, %1}, rd;\n\t}"
        : "=f"(d.x), "=f"(d.y)
        : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y), "f"(c.x), "f"(c.y));
    return d;
}
__device__ __forceinline__ float2 fadd2_rn(float2 a, float2 b) {
    float2 d;
    asm("{\n\t.reg .b64 ra, rb, rd;\n\t"
        "mov.b64 ra, {%2, %3};\n\tmov.b64 rb, {%4, %5};\n\t"
        "add.rn.f32x2 rd, ra, rb;\n\tmov.b64 {%0, %1}, rd;\n\t}"
        : "=f"(d.x), "=f"(d.y)
        : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y));
    return d;
}
__device__ __forceinline__ float2 fmul2_rn(float2 a, float2 b) {
    float2 d;
    asm("{\n\t.reg .b64 ra, rb, rd;\n\t"
        "mov.b64 ra, {%2, %3};\n\tmov.b64 rb, {%4, %5};\n\t"
        "mul.rn.f32x2 rd, ra, rb;\n\tmov.b64 {%0, %1}, rd;\n\t}"
        : "=f"(d.x), "=f"(d.y)
        : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y));
    return d;
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
// Per-token n x n parameters, prepared by lane groups.
//
// A warp is split into groups of GL lanes; each group owns one token, and
// lane q of a group holds elements e = q + GL * r (r < EPL) of the row-major
// n x n matrix, so every lane performs one (or two) of the n*n divisions of
// a pass in parallel. With one element per lane (n <= 5) a row or column sum
// gathers its n values with independent shuffles; with two (n = 6..8) it
// reads them from a small per-warp shared-memory buffer (kGroupScratch
// floats). Either way the n fetches of a sum overlap and the additions run
// in index order.
// ---------------------------------------------------------------------------
template <int N> struct Group {
    static constexpr int NN = N * N;
    static constexpr int GL = NN <= 1 ? 1 : NN <= 2 ? 2 : NN <= 4 ? 4 : NN <= 8 ? 8
                              : NN <= 16 ? 16 : 32;
    static constexpr int EPL = (NN + GL - 1) / GL;
    static constexpr int TPW = 32 / GL;  // tokens per warp
};
constexpr int kGroupScratch = 64;  // floats per warp: TPW * n * n <= 64 for n <= 8

// Sinkhorn projection of R independent batches of the warp's lane-group
// matrices (all 32 lanes call with the same K): M = exp(L); K times { divide
// every row by its sum; divide every column by its sum }. Sums run in index
// order starting from +0 and divisions are IEEE (__fdiv_rn), so every element
// sees a fixed sequence of correctly rounded operations. The R batches share
// the passes, so their latencies overlap. `scratch` holds R * kGroupScratch
// floats for this warp.
// SHFL selects how a lane gathers the n values of its row (column) when it
// owns one element (n <= 5): warp shuffles (shortest latency for one batch,
// the decode-sized calls) or the shared-memory buffer (more batches per unit
// time: the pipelined kernel's parameter warp, which must keep pace with the
// streams, measured faster on B200). Results are identical either way.
template <int N, int R, bool SHFL = true>
__device__ __forceinline__ void group_sinkhorn(float (&m)[R][Group<N>::EPL], float *scratch,
                                               int lane, int K) {
    constexpr int NN = N * N, GL = Group<N>::GL, EPL = Group<N>::EPL;
    const int q = lane & (GL - 1);
    int e[EPL], row[EPL], col[EPL];
    bool own[EPL];
#pragma unroll
    for (int r = 0; r < EPL; ++r) {
        e[r] = q + GL * r;
        own[r] = e[r] < NN;
        const int ec = own[r] ? e[r] : NN - 1;  // idle lanes shadow the last element
        row[r] = ec / N;
        col[r] = ec - row[r] * N;
    }
#pragma unroll
    for (int b = 0; b < R; ++b) {
#pragma unroll
        for (int r = 0; r < EPL; ++r) m[b][r] = expf(m[b][r]);
    }
    if constexpr (EPL == 1 && SHFL) {
        // one element per lane: the n values of a row (column) are fetched
        // with independent shuffles and added in index order
        const int base = lane & ~(GL - 1);
        for (int it = 0; it < K; ++it) {
#pragma unroll
            for (int pass = 0; pass < 2; ++pass) {
                float s[R];
#pragma unroll
                for (int b = 0; b < R; ++b) {
                    float v[N];
#pragma unroll
                    for (int k = 0; k < N; ++k)
                        v[k] = __shfl_sync(0xffffffffu, m[b][0],
                                           base + (pass == 0 ? row[0] * N + k : k * N + col[0]));
                    float acc = 0.0f;
#pragma unroll
                    for (int k = 0; k < N; ++k) acc = __fadd_rn(acc, v[k]);
                    s[b] = acc;
                }
#pragma unroll
                for (int b = 0; b < R; ++b) m[b][0] = __fdiv_rn(m[b][0], s[b]);
            }
        }
    } else {
        for (int it = 0; it < K; ++it) {
#pragma unroll
            for (int pass = 0; pass < 2; ++pass) {
#pragma unroll
                for (int b = 0; b < R; ++b) {
                    float *buf = scratch + b * kGroupScratch + (lane / GL) * NN;
#pragma unroll
                    for (int r = 0; r < EPL; ++r)
                        if (own[r]) buf[e[r]] = m[b][r];
                }
                __syncwarp();
                float s[R][EPL];
#pragma unroll
                for (int b = 0; b < R; ++b) {
                    const float *buf = scratch + b * kGroupScratch + (lane / GL) * NN;
#pragma unroll
                    for (int r = 0; r < EPL; ++r) {
                        float v[N];
#pragma unroll
                        for (int k = 0; k < N; ++k) v[k] = pass == 0 ? buf[row[r] * N + k] : buf[k * N + col[r]];
                        float acc = 0.0f;
#pragma unroll
                        for (int k = 0; k < N; ++k) acc = __fadd_rn(acc, v[k]);
                        s[b][r] = acc;
                    }
                }
                __syncwarp();
#pragma unroll
                for (int b = 0; b < R; ++b) {
#pragma unroll
                    for (int r = 0; r < EPL; ++r) m[b][r] = __fdiv_rn(m[b][r], s[b][r]);
                }
            }
        }
    }
}

// One batch (R = 1).
template <int N>
__device__ __forceinline__ void group_sinkhorn(float (&m)[Group<N>::EPL], float *scratch, int lane,
                                               int K) {
    float mm[1][Group<N>::EPL];
#pragma unroll
    for (int r = 0; r < Group<N>::EPL; ++r) mm[0][r] = m[r];
    group_sinkhorn<N, 1>(mm, scratch, lane, K);
#pragma unroll
    for (int r = 0; r < Group<N>::EPL; ++r) m[r] = mm[0][r];
}

// Softmax over the n read logits of the group's token. Lane q < N holds l_q
// on entry and a_q on exit; max and sum in index order.
template <int N>
__device__ __forceinline__ float group_softmax(float l, float *scratch, int lane) {
    constexpr int GL = Group<N>::GL;
    const int q = lane & (GL - 1);
    float *buf = scratch + (lane / GL) * N;
    if (q < N) buf[q] = l;
    __syncwarp();
    float v[N];
#pragma unroll
    for (int k = 0; k < N; ++k) v[k] = buf[k];
    __syncwarp();
    float mx = v[0];
#pragma unroll
    for (int k = 1; k < N; ++k)
        if (v[k] > mx) mx = v[k];
    float s = 0.0f;
#pragma unroll
    for (int k = 0; k < N; ++k) s = __fadd_rn(s, expf(__fsub_rn(v[k], mx)));
    return __fdiv_rn(expf(__fsub_rn(l, mx)), s);
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
// sequence (token of slot tt = first + tt * step): every warp takes TPW
// slots at a time with its lane groups. sA holds A row-major (row = source
// stream). `scratch` holds kGroupScratch floats per warp.
template <int N, bool WRITE, bool READ>
__device__ __forceinline__ void prepare_params(const StepParams &p, int64_t first, int64_t step,
                                               int TB, float *sA, float *sb, float *sa,
                                               float *scratch) {
    constexpr int NN = N * N, GL = Group<N>::GL, EPL = Group<N>::EPL, TPW = Group<N>::TPW;
    const int lane = threadIdx.x & 31;
    const int warp = threadIdx.x >> 5;
    const int nwarps = blockDim.x >> 5;
    const int q = lane & (GL - 1);
    float *wscratch = scratch + warp * kGroupScratch;
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
            if (p.mix_logits) group_sinkhorn<N>(m, wscratch, lane, p.K);  // warp-uniform branch
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
            if (p.read_logits) l = group_softmax<N>(l, wscratch, lane);
            if (live && q < N) sa[tt * N + q] = l;
        }
    }
}

}  // namespace hc
