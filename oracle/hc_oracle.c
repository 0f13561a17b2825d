/*
 * hc_oracle.c -- plain, slow CPU oracle for the Hyper-Connections residual step.
 *
 * TEST INFRASTRUCTURE. Only the test suite, the package smoke check and the
 * benchmark's CPU-baseline / reference arm may load this library. The product
 * path (the CUDA library under hyper_connections_stream_b200/) never calls it,
 * and this file includes nothing from there: no header, helper, table or
 * kernel is shared.
 *
 * What it computes (sources are the pages' titles and sections):
 *  - "Hyper-connections (mHC)" glossary entry (hfviewer), definition paragraph:
 *    the residual stream is widened to n parallel streams, learned matrices mix
 *    the streams before the block (read) and after it (write), and the mHC
 *    variant makes the mixing doubly stochastic with a few Sinkhorn iterations.
 *  - "Tencent open-sources Hy4 Preview at 770B -- Identity Hyper-Connections"
 *    (learnaivisually), Jargon ("Pre-norm", "Identity initialization") and the
 *    TL;DR: the block normalises its input (pre-norm), n = 4 streams, and an
 *    untrained HC network computes exactly what a one-stream network computes.
 *
 * The pages print no equations. The readings used here (all stated again in
 * the design notes):
 *  - write:  H'_j = sum_i A[i][j] * H_i + b_j * y   (row i = source stream,
 *            column j = destination stream)
 *  - read:   h = sum_i a_i * H_i, then x = RMSNorm(h) * g (pre-norm of the
 *            next block; eps inside the square root, per-channel gain g)
 *  - Sinkhorn: M = exp(L) (no max shift); then K times: divide every row by
 *            its sum, then every column by its sum. Exactly K row+column pairs,
 *            no early exit.
 *  - read-weight softmax (mHC): a_i = exp(l_i - max l) / sum_k exp(l_k - max l)
 *
 * Arithmetic (fp32 accumulation, storage dtype rounding, as the workload fixes):
 *  - every multiply-add is a correctly rounded fp32 fused multiply-add (fmaf),
 *    chained in stream order i = 0..n-1, starting from -0.0f (the neutral
 *    element of IEEE addition, so the first step is just the rounded product);
 *  - storage rounding (fp32 -> bf16, round to nearest even) happens only where
 *    a result is stored: H', x and the harness's block output y;
 *  - the RMSNorm statistic is accumulated in fp64 (squares of fp32 values are
 *    exact in fp64), r = (float)(1 / sqrt(ss / d + eps)) is rounded once, and
 *    x = (h * r) * g is two fp32 multiplies;
 *  - sums inside the Sinkhorn projection and the softmax run in index order.
 * Compiled with -ffp-contract=off so that no other fused operation appears.
 *
 * Tokens are independent, so each entry point loops over tokens with an
 * OpenMP parallel-for; the arithmetic of a token does not depend on the
 * thread count.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

#define HCO_F32 0
#define HCO_BF16 1

#define HCO_OK 0
#define HCO_EINVAL 1

/* ---- storage dtype helpers (the oracle's own; bf16 is the top half of fp32) */

static float bf16_bits_to_f32(uint16_t v) {
    uint32_t u = (uint32_t)v << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return f;
}

/* fp32 -> bf16, round to nearest, ties to even. NaN stays NaN (quiet). */
static uint16_t f32_to_bf16_bits(float f) {
    uint32_t u;
    memcpy(&u, &f, sizeof u);
    if ((u & 0x7f800000u) == 0x7f800000u && (u & 0x007fffffu) != 0u)
        return (uint16_t)((u >> 16) | 0x0040u);
    uint32_t lower = u & 0xffffu;
    uint32_t upper = u >> 16;
    if (lower > 0x8000u || (lower == 0x8000u && (upper & 1u)))
        upper += 1u; /* a carry into the exponent is the correct rounding */
    return (uint16_t)upper;
}

static float load_s(const void *p, int dt, int64_t i) {
    if (dt == HCO_BF16) return bf16_bits_to_f32(((const uint16_t *)p)[i]);
    return ((const float *)p)[i];
}

static void store_s(void *p, int dt, int64_t i, float v) {
    if (dt == HCO_BF16)
        ((uint16_t *)p)[i] = f32_to_bf16_bits(v);
    else
        ((float *)p)[i] = v;
}

/* Value a storage slot would hold after storing v (the rounding alone). */
static float round_s(int dt, float v) {
    if (dt == HCO_BF16) return bf16_bits_to_f32(f32_to_bf16_bits(v));
    return v;
}

/* ---- (mHC) Sinkhorn projection of one n x n logit matrix, fp32 ---------- */

static void sinkhorn_one_f32(const float *L, float *M, int n, int K) {
    for (int e = 0; e < n * n; ++e) M[e] = expf(L[e]);
    for (int k = 0; k < K; ++k) {
        for (int i = 0; i < n; ++i) { /* row pass: every row sums to 1 */
            float s = 0.0f;
            for (int j = 0; j < n; ++j) s = s + M[i * n + j];
            for (int j = 0; j < n; ++j) M[i * n + j] = M[i * n + j] / s;
        }
        for (int j = 0; j < n; ++j) { /* column pass: every column sums to 1 */
            float s = 0.0f;
            for (int i = 0; i < n; ++i) s = s + M[i * n + j];
            for (int i = 0; i < n; ++i) M[i * n + j] = M[i * n + j] / s;
        }
    }
}

/* Same projection in fp64 (used by the invariant checks, not by the step). */
static void sinkhorn_one_f64(const double *L, double *M, int n, int K) {
    for (int e = 0; e < n * n; ++e) M[e] = exp(L[e]);
    for (int k = 0; k < K; ++k) {
        for (int i = 0; i < n; ++i) {
            double s = 0.0;
            for (int j = 0; j < n; ++j) s = s + M[i * n + j];
            for (int j = 0; j < n; ++j) M[i * n + j] = M[i * n + j] / s;
        }
        for (int j = 0; j < n; ++j) {
            double s = 0.0;
            for (int i = 0; i < n; ++i) s = s + M[i * n + j];
            for (int i = 0; i < n; ++i) M[i * n + j] = M[i * n + j] / s;
        }
    }
}

/* ---- (mHC) read weights: softmax over the n streams --------------------- */

static void softmax_one_f32(const float *l, float *a, int n) {
    float mx = l[0];
    for (int i = 1; i < n; ++i)
        if (l[i] > mx) mx = l[i];
    float s = 0.0f;
    for (int i = 0; i < n; ++i) {
        a[i] = expf(l[i] - mx);
        s = s + a[i];
    }
    for (int i = 0; i < n; ++i) a[i] = a[i] / s;
}

/* ---- write mix for one token: H'_j = sum_i A[i][j] H_i + b_j y ---------- */

static void write_token(const void *H, const void *y, void *Hout, int dt, int n,
                        int64_t d, int64_t t, const float *A, const float *b) {
    float out[16];
    for (int64_t k = 0; k < d; ++k) {
        float yk = load_s(y, dt, t * d + k);
        for (int j = 0; j < n; ++j) {
            float acc = -0.0f;
            for (int i = 0; i < n; ++i)
                acc = fmaf(A[i * n + j], load_s(H, dt, (t * n + i) * d + k), acc);
            acc = fmaf(b[j], yk, acc);
            out[j] = acc;
        }
        /* all n outputs of this element are formed before any is stored, so
         * Hout may be the same buffer as H */
        for (int j = 0; j < n; ++j) store_s(Hout, dt, (t * n + j) * d + k, out[j]);
    }
}

/* ---- RMSNorm of one fp32 row h[d] into storage x[d] ---------------------- */

static void rmsnorm_row(const float *h, void *x, int dt, int64_t d, int64_t x_off,
                        const float *g, float eps) {
    double ss = 0.0;
    for (int64_t k = 0; k < d; ++k) ss += (double)h[k] * (double)h[k];
    float r = (float)(1.0 / sqrt(ss / (double)d + (double)eps));
    for (int64_t k = 0; k < d; ++k) {
        float v = h[k] * r;
        v = v * (g ? g[k] : 1.0f);
        store_s(x, dt, x_off + k, v);
    }
}

/* ---- read mix + pre-norm for one token: x = RMSNorm(sum_i a_i H_i) * g --- */

static void read_token(const void *H, void *x, int dt, int n, int64_t d, int64_t t,
                       const float *a, const float *g, float eps, float *hbuf) {
    for (int64_t k = 0; k < d; ++k) {
        float acc = -0.0f;
        for (int i = 0; i < n; ++i) acc = fmaf(a[i], load_s(H, dt, (t * n + i) * d + k), acc);
        hbuf[k] = acc;
    }
    rmsnorm_row(hbuf, x, dt, d, t * d, g, eps);
}

static int check_common(int dt, int64_t T, int n, int64_t d) {
    if (dt != HCO_F32 && dt != HCO_BF16) return HCO_EINVAL;
    if (T < 0 || n < 1 || n > 16 || d < 1) return HCO_EINVAL;
    return HCO_OK;
}

/* Per-token parameter pointers: stride 0 = one set for every token. */
static const float *tok_ptr(const float *p, int64_t stride, int64_t t) {
    return p ? p + stride * t : NULL;
}

/* =========================== exported entry points ======================== */

int hco_max_threads(void) {
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

void hco_set_threads(int nthreads) {
#ifdef _OPENMP
    if (nthreads > 0) omp_set_num_threads(nthreads);
#else
    (void)nthreads;
#endif
}

/* storage rounding of a buffer of fp32 values into dtype dt */
int hco_round_to(const float *src, void *dst, int dt, int64_t count) {
    if (dt != HCO_F32 && dt != HCO_BF16) return HCO_EINVAL;
    for (int64_t i = 0; i < count; ++i) store_s(dst, dt, i, src[i]);
    return HCO_OK;
}

int hco_sinkhorn_f32(const float *L, float *out, int64_t T, int n, int K) {
    if (T < 0 || n < 1 || n > 16 || K < 0) return HCO_EINVAL;
#pragma omp parallel for schedule(static)
    for (int64_t t = 0; t < T; ++t) sinkhorn_one_f32(L + t * n * n, out + t * n * n, n, K);
    return HCO_OK;
}

int hco_sinkhorn_f64(const double *L, double *out, int64_t T, int n, int K) {
    if (T < 0 || n < 1 || n > 16 || K < 0) return HCO_EINVAL;
#pragma omp parallel for schedule(static)
    for (int64_t t = 0; t < T; ++t) sinkhorn_one_f64(L + t * n * n, out + t * n * n, n, K);
    return HCO_OK;
}

int hco_softmax_f32(const float *l, float *a, int64_t T, int n) {
    if (T < 0 || n < 1 || n > 16) return HCO_EINVAL;
#pragma omp parallel for schedule(static)
    for (int64_t t = 0; t < T; ++t) softmax_one_f32(l + t * n, a + t * n, n);
    return HCO_OK;
}

/* Write mix with the mixing matrix given (A, stride A_s floats per token). */
int hco_write_mix(const void *H, const void *y, void *Hout, int dt, int64_t T, int n,
                  int64_t d, const float *A, int64_t A_s, const float *b, int64_t b_s) {
    if (check_common(dt, T, n, d) || !A || !b) return HCO_EINVAL;
#pragma omp parallel for schedule(static)
    for (int64_t t = 0; t < T; ++t)
        write_token(H, y, Hout, dt, n, d, t, tok_ptr(A, A_s, t), tok_ptr(b, b_s, t));
    return HCO_OK;
}

/* Read mix + RMSNorm with the read weights given (a, stride a_s per token).
 * g may be NULL (gain 1). */
int hco_read_rmsnorm(const void *H, void *x, int dt, int64_t T, int n, int64_t d,
                     const float *a, int64_t a_s, const float *g, float eps) {
    if (check_common(dt, T, n, d) || !a) return HCO_EINVAL;
    int err = HCO_OK;
#pragma omp parallel
    {
        float *hbuf = (float *)malloc(sizeof(float) * (size_t)d);
        if (!hbuf) {
#pragma omp atomic write
            err = HCO_EINVAL;
        } else {
#pragma omp for schedule(static)
            for (int64_t t = 0; t < T; ++t)
                read_token(H, x, dt, n, d, t, tok_ptr(a, a_s, t), g, eps, hbuf);
        }
        free(hbuf);
    }
    return err;
}

/*
 * One HC residual step as a single operation: layer l's write followed by
 * layer l+1's read, reading the *stored* (rounded) H'.
 *   mix_logits != 0: A holds logits, projected per token by K Sinkhorn pairs.
 *   read_logits != 0: a holds logits, turned into weights by a softmax.
 * Hout may equal H. x_next must not overlap H or Hout.
 */
int hco_write_then_read(const void *H, const void *y, void *Hout, void *x_next, int dt,
                        int64_t T, int n, int64_t d, int mix_logits, const float *A,
                        int64_t A_s, int K, const float *b, int64_t b_s, int read_logits,
                        const float *a, int64_t a_s, const float *g, float eps) {
    if (check_common(dt, T, n, d) || !A || !b || !a || (mix_logits && K < 0))
        return HCO_EINVAL;
    int err = HCO_OK;
#pragma omp parallel
    {
        float *hbuf = (float *)malloc(sizeof(float) * (size_t)d);
        float Am[256], aw[16];
        if (!hbuf) {
#pragma omp atomic write
            err = HCO_EINVAL;
        } else {
#pragma omp for schedule(static)
            for (int64_t t = 0; t < T; ++t) {
                const float *At = tok_ptr(A, A_s, t);
                const float *at = tok_ptr(a, a_s, t);
                if (mix_logits) {
                    sinkhorn_one_f32(At, Am, n, K);
                    At = Am;
                }
                if (read_logits) {
                    softmax_one_f32(at, aw, n);
                    at = aw;
                }
                write_token(H, y, Hout, dt, n, d, t, At, tok_ptr(b, b_s, t));
                read_token(Hout, x_next, dt, n, d, t, at, g, eps, hbuf);
            }
        }
        free(hbuf);
    }
    return err;
}

/*
 * Input-dependent mixing logits (the step's per-token parameters computed from
 * the streams themselves; the glossary entry only says the mixing matrices are
 * learned). Reading: u = the token's n*d stream values flattened, r = 1 /
 * sqrt(mean(u^2) + eps), z[j] = r * sum_k u[k] * W[j][k] for j < P.
 * W is [P][n*d] in storage dtype dt (row j = the weights of logit j).
 * Computed in fp64 (no rounding but the final one to fp64), as a reference.
 */
int hco_mix_logits(const void *H, const void *W, double *z, int dt, int64_t T, int n, int64_t d,
                   int P, float eps) {
    if (check_common(dt, T, n, d) || P < 1) return HCO_EINVAL;
    const int64_t K = (int64_t)n * d;
#pragma omp parallel for schedule(static)
    for (int64_t t = 0; t < T; ++t) {
        double ss = 0.0;
        for (int64_t k = 0; k < K; ++k) {
            const double u = (double)load_s(H, dt, t * K + k);
            ss += u * u;
        }
        const double r = 1.0 / sqrt(ss / (double)K + (double)eps);
        for (int j = 0; j < P; ++j) {
            double acc = 0.0;
            for (int64_t k = 0; k < K; ++k)
                acc += (double)load_s(H, dt, t * K + k) * (double)load_s(W, dt, (int64_t)j * K + k);
            z[t * P + j] = r * acc;
        }
    }
    return HCO_OK;
}

/*
 * Ends of a stack ("Tencent open-sources Hy4 Preview at 770B -- Identity
 * Hyper-Connections", learnaivisually: TL;DR and the residual-design table,
 * the n streams start as copies of one). Expansion: every stream of token t
 * is a copy of x[t]. The pages do not say how the streams are combined at the
 * top; reading: a weighted sum of the streams, out = sum_i w_i H_i, the same
 * fmaf chain in stream order as the read mix, stored without normalisation.
 */
int hco_expand(const void *x, void *H, int dt, int64_t T, int n, int64_t d) {
    if (check_common(dt, T, n, d)) return HCO_EINVAL;
#pragma omp parallel for schedule(static)
    for (int64_t t = 0; t < T; ++t)
        for (int i = 0; i < n; ++i)
            for (int64_t k = 0; k < d; ++k)
                store_s(H, dt, (t * n + i) * d + k, load_s(x, dt, t * d + k));
    return HCO_OK;
}

int hco_collapse(const void *H, void *out, int dt, int64_t T, int n, int64_t d, int read_logits,
                 const float *w, int64_t w_s) {
    if (check_common(dt, T, n, d) || !w) return HCO_EINVAL;
#pragma omp parallel for schedule(static)
    for (int64_t t = 0; t < T; ++t) {
        float ww[16];
        const float *wt = tok_ptr(w, w_s, t);
        if (read_logits) {
            softmax_one_f32(wt, ww, n);
            wt = ww;
        }
        for (int64_t k = 0; k < d; ++k) {
            float acc = -0.0f;
            for (int i = 0; i < n; ++i) acc = fmaf(wt[i], load_s(H, dt, (t * n + i) * d + k), acc);
            store_s(out, dt, t * d + k, acc);
        }
    }
    return HCO_OK;
}

/*
 * The block's output projection (a plain linear map), as a reference for the
 * fused projection + write: y[t][c] = sum_k X[t][k] * W[c][k], W one row per
 * output channel. Computed in fp64 (products of bf16 or fp32 values are exact
 * in fp64; sums in index order), stored as fp64. Not part of the HC step
 * itself: the write mix of a given y is hco_write_mix.
 */
int hco_linear(const void *X, const void *W, double *y, int dt, int64_t T, int64_t k, int64_t d) {
    if ((dt != HCO_F32 && dt != HCO_BF16) || T < 0 || k < 1 || d < 1) return HCO_EINVAL;
#pragma omp parallel for schedule(static)
    for (int64_t t = 0; t < T; ++t)
        for (int64_t c = 0; c < d; ++c) {
            double acc = 0.0;
            for (int64_t kk = 0; kk < k; ++kk)
                acc += (double)load_s(X, dt, t * k + kk) * (double)load_s(W, dt, c * k + kk);
            y[t * d + c] = acc;
        }
    return HCO_OK;
}

/*
 * Backward pass of the fused step (training). The forward is hco_write_then_read;
 * storage rounding is treated as the identity for gradients (its derivative
 * almost everywhere), so the gradients are those of the exact-arithmetic step
 * evaluated at the stored forward values (H' as stored, h as the fp32 chain,
 * r as rounded to fp32). All backward arithmetic is fp64:
 *   x_k  = h_k r g_k,  r = (sum h^2 / d + eps)^(-1/2)
 *   dh_k = r g_k dx_k - (r^3 / d) h_k sum_m g_m dx_m h_m      (RMSNorm)
 *   dg_k = sum_t dx_k h_k r                                  (over tokens)
 *   G_j  = dH'_j + a_j dh                                    (into stream j of H')
 *   dH_i = sum_j A[i][j] G_j,  dy = sum_j b_j G_j
 *   dA[i][j] = sum_k H_i,k G_j,k,  db_j = sum_k y_k G_j,k,  da_j = sum_k dh_k H'_j,k
 * then, per token, through the softmax of the read logits
 *   dl_j = a_j (da_j - sum_m a_m da_m)
 * and through the Sinkhorn projection: the K (row, column) pairs are re-run
 * in fp64 keeping every intermediate, then each normalisation M' = M / s is
 * undone in reverse order with dM = (dM' - sum(dM' * M') over the same row or
 * column) / s, and finally dL = dM * exp(L).
 * dHout may be NULL (no gradient arrives at H'); dg may be NULL.
 */
static void sinkhorn_backward_f64(const float *L, const double *dA, double *dL, int n, int K,
                                  double *hist /* (2K+1) n*n */) {
    const int nn = n * n;
    for (int e = 0; e < nn; ++e) hist[e] = exp((double)L[e]);
    for (int p = 0; p < 2 * K; ++p) {
        const double *in = hist + (int64_t)p * nn;
        double *out = hist + (int64_t)(p + 1) * nn;
        for (int q = 0; q < n; ++q) {
            double s = 0.0;
            for (int k = 0; k < n; ++k) s += (p % 2 == 0) ? in[q * n + k] : in[k * n + q];
            for (int k = 0; k < n; ++k) {
                const int e = (p % 2 == 0) ? q * n + k : k * n + q;
                out[e] = in[e] / s;
            }
        }
    }
    double gcur[256], gnext[256];
    for (int e = 0; e < nn; ++e) gcur[e] = dA[e];
    for (int p = 2 * K - 1; p >= 0; --p) {
        const double *in = hist + (int64_t)p * nn;
        const double *out = hist + (int64_t)(p + 1) * nn;
        for (int q = 0; q < n; ++q) {
            double s = 0.0, t = 0.0;
            for (int k = 0; k < n; ++k) {
                const int e = (p % 2 == 0) ? q * n + k : k * n + q;
                s += in[e];
                t += gcur[e] * out[e];
            }
            for (int k = 0; k < n; ++k) {
                const int e = (p % 2 == 0) ? q * n + k : k * n + q;
                gnext[e] = (gcur[e] - t) / s;
            }
        }
        for (int e = 0; e < nn; ++e) gcur[e] = gnext[e];
    }
    for (int e = 0; e < nn; ++e) dL[e] = gcur[e] * hist[e];
}

int hco_sinkhorn_backward(const float *L, const double *dA, double *dL, int64_t T, int n, int K) {
    if (T < 0 || n < 1 || n > 16 || K < 0) return HCO_EINVAL;
    int err = HCO_OK;
#pragma omp parallel
    {
        double *hist = (double *)malloc(sizeof(double) * (size_t)(2 * K + 1) * (size_t)(n * n));
        if (!hist) {
#pragma omp atomic write
            err = HCO_EINVAL;
        } else {
#pragma omp for schedule(static)
            for (int64_t t = 0; t < T; ++t)
                sinkhorn_backward_f64(L + t * n * n, dA + t * n * n, dL + t * n * n, n, K, hist);
        }
        free(hist);
    }
    return err;
}

int hco_write_then_read_backward(const void *H, const void *y, int dt, int64_t T, int n, int64_t d,
                                 int mix_logits, const float *A, int64_t A_s, int K, const float *b,
                                 int64_t b_s, int read_logits, const float *a, int64_t a_s,
                                 const float *g, float eps, const double *dHout, const double *dx,
                                 double *dH, double *dy, double *dA, double *db, double *da,
                                 double *dg) {
    if (check_common(dt, T, n, d) || !A || !b || !a || !dx || (mix_logits && K < 0) || n > 8)
        return HCO_EINVAL;
    int err = HCO_OK;
    const int nt = omp_get_max_threads();
    double *dg_part = dg ? (double *)calloc((size_t)nt * (size_t)d, sizeof(double)) : NULL;
    if (dg && !dg_part) return HCO_EINVAL;
#pragma omp parallel
    {
        const int tid = omp_get_thread_num();
        float *Hs = (float *)malloc(sizeof(float) * (size_t)n * (size_t)d);
        float *h = (float *)malloc(sizeof(float) * (size_t)d);
        double *dh = (double *)malloc(sizeof(double) * (size_t)d);
        double *hist = (double *)malloc(sizeof(double) * (size_t)(2 * (K > 0 ? K : 0) + 1) * 64);
        if (!Hs || !h || !dh || !hist) {
#pragma omp atomic write
            err = HCO_EINVAL;
        } else {
#pragma omp for schedule(static)
            for (int64_t t = 0; t < T; ++t) {
                float Am[64], aw[8];
                const float *At = tok_ptr(A, A_s, t), *bt = tok_ptr(b, b_s, t), *at = tok_ptr(a, a_s, t);
                if (mix_logits) {
                    sinkhorn_one_f32(At, Am, n, K);
                    At = Am;
                }
                if (read_logits) {
                    softmax_one_f32(at, aw, n);
                    at = aw;
                }
                /* forward values as the forward stores / computes them */
                for (int64_t k = 0; k < d; ++k) {
                    const float yk = load_s(y, dt, t * d + k);
                    float hk = -0.0f;
                    for (int j = 0; j < n; ++j) {
                        float acc = -0.0f;
                        for (int i = 0; i < n; ++i)
                            acc = fmaf(At[i * n + j], load_s(H, dt, (t * n + i) * d + k), acc);
                        acc = fmaf(bt[j], yk, acc);
                        Hs[j * d + k] = round_s(dt, acc);
                        hk = fmaf(at[j], Hs[j * d + k], hk);
                    }
                    h[k] = hk;
                }
                double ss = 0.0;
                for (int64_t k = 0; k < d; ++k) ss += (double)h[k] * (double)h[k];
                const double r = (double)(float)(1.0 / sqrt(ss / (double)d + (double)eps));
                /* RMSNorm backward */
                double sg = 0.0;
                for (int64_t k = 0; k < d; ++k) sg += (g ? (double)g[k] : 1.0) * dx[t * d + k] * (double)h[k];
                for (int64_t k = 0; k < d; ++k) {
                    const double gk = g ? (double)g[k] : 1.0;
                    dh[k] = r * gk * dx[t * d + k] - r * r * r / (double)d * (double)h[k] * sg;
                    if (dg_part) dg_part[(int64_t)tid * d + k] += dx[t * d + k] * (double)h[k] * r;
                }
                /* mixes */
                double gA[64] = {0}, gb[8] = {0}, ga[8] = {0};
                for (int64_t k = 0; k < d; ++k) {
                    double G[8];
                    const double yk = (double)load_s(y, dt, t * d + k);
                    for (int j = 0; j < n; ++j) {
                        G[j] = (dHout ? dHout[(t * n + j) * d + k] : 0.0) + (double)at[j] * dh[k];
                        gb[j] += yk * G[j];
                        ga[j] += dh[k] * (double)Hs[j * d + k];
                    }
                    double dyk = 0.0;
                    for (int j = 0; j < n; ++j) dyk += (double)bt[j] * G[j];
                    dy[t * d + k] = dyk;
                    for (int i = 0; i < n; ++i) {
                        const double hik = (double)load_s(H, dt, (t * n + i) * d + k);
                        double acc = 0.0;
                        for (int j = 0; j < n; ++j) {
                            acc += (double)At[i * n + j] * G[j];
                            gA[i * n + j] += hik * G[j];
                        }
                        dH[(t * n + i) * d + k] = acc;
                    }
                }
                for (int j = 0; j < n; ++j) db[t * n + j] = gb[j];
                if (read_logits) {
                    double sa = 0.0;
                    for (int j = 0; j < n; ++j) sa += (double)at[j] * ga[j];
                    for (int j = 0; j < n; ++j) da[t * n + j] = (double)at[j] * (ga[j] - sa);
                } else {
                    for (int j = 0; j < n; ++j) da[t * n + j] = ga[j];
                }
                if (mix_logits)
                    sinkhorn_backward_f64(tok_ptr(A, A_s, t), gA, dA + t * n * n, n, K, hist);
                else
                    for (int e = 0; e < n * n; ++e) dA[t * n * n + e] = gA[e];
            }
        }
        free(Hs);
        free(h);
        free(dh);
        free(hist);
    }
    if (dg) {
        for (int64_t k = 0; k < d; ++k) {
            double acc = 0.0;
            for (int q = 0; q < nt; ++q) acc += dg_part[(int64_t)q * d + k];
            dg[k] = acc;
        }
        free(dg_part);
    }
    return err;
}

/* Harness block stand-in: y = round_s(tanhf(x)). Not part of the HC step. */
int hco_block_tanh(const void *x, void *y, int dt, int64_t count) {
    if (dt != HCO_F32 && dt != HCO_BF16) return HCO_EINVAL;
#pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < count; ++i) store_s(y, dt, i, tanhf(load_s(x, dt, i)));
    return HCO_OK;
}

/*
 * The ordinary one-stream pre-norm residual layer that HC replaces:
 *   x_out = round_s(x + round_s(tanh(RMSNorm(x) * g)))
 * where RMSNorm(x) * g is stored (rounded) before the tanh, exactly as the HC
 * path stores its block input. Used to check the identity initialisation.
 */
int hco_single_stream_layer(const void *x, void *x_out, int dt, int64_t T, int64_t d,
                            const float *g, float eps) {
    if (check_common(dt, T, 1, d)) return HCO_EINVAL;
    int err = HCO_OK;
#pragma omp parallel
    {
        float *h = (float *)malloc(sizeof(float) * (size_t)d);
        float *xn = (float *)malloc(sizeof(float) * (size_t)d);
        if (!h || !xn) {
#pragma omp atomic write
            err = HCO_EINVAL;
        } else {
#pragma omp for schedule(static)
            for (int64_t t = 0; t < T; ++t) {
                for (int64_t k = 0; k < d; ++k) h[k] = load_s(x, dt, t * d + k);
                rmsnorm_row(h, xn, HCO_F32, d, 0, g, eps);
                for (int64_t k = 0; k < d; ++k) {
                    float normed = round_s(dt, xn[k]);
                    float yk = round_s(dt, tanhf(normed));
                    store_s(x_out, dt, t * d + k, h[k] + yk);
                }
            }
        }
        free(h);
        free(xn);
    }
    return err;
}
