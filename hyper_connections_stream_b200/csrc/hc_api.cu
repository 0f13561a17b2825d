// hc_api.cu -- host side of libhc_b200.so: argument validation, launch
// configuration and error reporting for the HC step kernels (the C ABI is
// declared in include/hc_api.h).
//
// Nothing here allocates device memory or synchronises; every launch goes on
// the caller's stream.

#include <cuda_runtime.h>

#include <climits>
#include <cmath>
#include <cstdarg>
#include <cstdio>
#include <cstring>

#include "hc_api.h"
#include "hc_stream_kernels.cuh"

namespace {

thread_local char g_last_error[512] = "";

hc_status fail(hc_status st, const char *fmt, ...) {
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(g_last_error, sizeof g_last_error, fmt, ap);
    va_end(ap);
    return st;
}

hc_status check_launch(const char *what) {
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess)
        return fail(HC_ERR_CUDA, "%s: launch failed: %s", what, cudaGetErrorString(e));
    return HC_OK;
}

bool aligned(const void *p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

bool overlap(const void *p, int64_t pb, const void *q, int64_t qb) {
    if (!p || !q || pb <= 0 || qb <= 0) return false;
    const uintptr_t a0 = reinterpret_cast<uintptr_t>(p), a1 = a0 + (uintptr_t)pb;
    const uintptr_t b0 = reinterpret_cast<uintptr_t>(q), b1 = b0 + (uintptr_t)qb;
    return a0 < b1 && b0 < a1;
}

int elem_bytes(hc_dtype dt) { return dt == HC_BF16 ? 2 : 4; }
int vec_elems(hc_dtype dt) { return dt == HC_BF16 ? 8 : 4; }

struct DeviceInfo {
    int sms = 0;
};

hc_status device_info(DeviceInfo &info) {
    static DeviceInfo cache[64];
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return fail(HC_ERR_CUDA, "cudaGetDevice: %s", cudaGetErrorString(e));
    if (dev < 0 || dev >= 64) return fail(HC_ERR_UNSUPPORTED, "device ordinal %d >= 64", dev);
    if (cache[dev].sms == 0) {
        int sms = 0;
        e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
        if (e != cudaSuccess)
            return fail(HC_ERR_CUDA, "cudaDeviceGetAttribute: %s", cudaGetErrorString(e));
        cache[dev].sms = sms;
    }
    info = cache[dev];
    return HC_OK;
}

// ---- common validation -----------------------------------------------------

struct Shape {
    hc_dtype dt;
    int64_t T;
    int n;
    int64_t d;
};

hc_status check_shape(const char *fn, const Shape &s, bool normalises) {
    if (s.dt != HC_F32 && s.dt != HC_BF16) return fail(HC_ERR_INVALID_ARG, "%s: bad dtype %d", fn, (int)s.dt);
    if (s.T < 0) return fail(HC_ERR_INVALID_ARG, "%s: T = %lld < 0", fn, (long long)s.T);
    if (s.n < 1) return fail(HC_ERR_INVALID_ARG, "%s: n = %d < 1", fn, s.n);
    if (s.n > hc::kMaxStreams) return fail(HC_ERR_UNSUPPORTED, "%s: n = %d > %d", fn, s.n, hc::kMaxStreams);
    if (s.d < 1) return fail(HC_ERR_INVALID_ARG, "%s: d = %lld < 1", fn, (long long)s.d);
    if (s.d % vec_elems(s.dt) != 0)
        return fail(HC_ERR_UNSUPPORTED, "%s: d = %lld is not a multiple of %d (16-byte vectors)", fn,
                    (long long)s.d, vec_elems(s.dt));
    const int64_t dmax = (int64_t)hc::kStreamMaxThreads * 8 * vec_elems(s.dt);
    if (normalises && s.d > dmax)
        return fail(HC_ERR_UNSUPPORTED, "%s: d = %lld > %lld for a normalising call", fn,
                    (long long)s.d, (long long)dmax);
    // byte sizes must fit in int64
    const int64_t row = (int64_t)s.n * s.d * elem_bytes(s.dt);
    if (s.T > 0 && s.T > INT64_MAX / row) return fail(HC_ERR_INVALID_ARG, "%s: T*n*d overflows", fn);
    return HC_OK;
}

hc_status check_stride(const char *fn, const char *name, int64_t stride) {
    if (stride < 0) return fail(HC_ERR_INVALID_ARG, "%s: %s = %lld < 0", fn, name, (long long)stride);
    return HC_OK;
}

hc_status check_param(const char *fn, const char *name, const float *p) {
    if (!p) return fail(HC_ERR_INVALID_ARG, "%s: %s is NULL", fn, name);
    if (!aligned(p, 4)) return fail(HC_ERR_MISALIGNED, "%s: %s is not 4-byte aligned", fn, name);
    return HC_OK;
}

hc_status check_buf(const char *fn, const char *name, const void *p) {
    if (!p) return fail(HC_ERR_INVALID_ARG, "%s: %s is NULL", fn, name);
    if (!aligned(p, 16)) return fail(HC_ERR_MISALIGNED, "%s: %s is not 16-byte aligned", fn, name);
    return HC_OK;
}

hc_status check_eps(const char *fn, float eps) {
    if (!(eps >= 0.0f) || std::isinf(eps))
        return fail(HC_ERR_INVALID_ARG, "%s: eps must be finite and >= 0", fn);
    return HC_OK;
}

hc_status check_K(const char *fn, int K) {
    if (K < 1) return fail(HC_ERR_INVALID_ARG, "%s: K = %d < 1", fn, K);
    if (K > (1 << 16)) return fail(HC_ERR_UNSUPPORTED, "%s: K = %d > 65536", fn, K);
    return HC_OK;
}

#define HC_TRY(expr)                       \
    do {                                   \
        hc_status _st = (expr);            \
        if (_st != HC_OK) return _st;      \
    } while (0)

// ---- launch of the streaming kernels -----------------------------------------

template <int N, typename S, int KIND, int CPT>
hc_status launch_stream_cpt(const hc::StepParams &p, int NT, int sms, cudaStream_t st) {
    auto kern = hc::hc_stream_kernel<N, S, KIND, CPT>;
    int per_sm = 0;
    cudaError_t e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, NT, 0);
    if (e != cudaSuccess) return fail(HC_ERR_CUDA, "occupancy query: %s", cudaGetErrorString(e));
    if (per_sm < 1) per_sm = 1;
    int64_t grid = (int64_t)sms * per_sm;
    if (grid > p.T) grid = p.T;
    kern<<<(unsigned)grid, NT, 0, st>>>(p);
    return check_launch("hc_stream_kernel");
}

// Pick threads per CTA (NT) and 16-byte slices per thread (CPT) for a row of
// nvec slices: the smallest CPT whose NT fits, preferring no idle slices.
void pick_stream_shape(int64_t nvec, bool normalises, int &NT, int &CPT) {
    if (!normalises) {
        // no per-thread state: one pass of up to 256 threads over the row
        int64_t t = nvec < 256 ? nvec : 256;
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
        if (nt > hc::kStreamMaxThreads) continue;
        if (nt < 64 && cpt > 1) continue;  // fewer slices per thread is better here
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
hc_status launch_stream(const hc::StepParams &p, cudaStream_t st) {
    DeviceInfo info;
    HC_TRY(device_info(info));
    constexpr int V = hc::StorageTraits<S>::V;
    const int64_t nvec = p.d / V;
    int NT = 0, CPT = 1;
    pick_stream_shape(nvec, KIND != hc::KIND_WRITE, NT, CPT);
    if (NT == 0) return fail(HC_ERR_UNSUPPORTED, "no launch shape for d = %lld", (long long)p.d);
    if constexpr (KIND == hc::KIND_WRITE) {
        return launch_stream_cpt<N, S, KIND, 1>(p, NT, info.sms, st);
    } else {
        switch (CPT) {
            case 1: return launch_stream_cpt<N, S, KIND, 1>(p, NT, info.sms, st);
            case 2: return launch_stream_cpt<N, S, KIND, 2>(p, NT, info.sms, st);
            case 4: return launch_stream_cpt<N, S, KIND, 4>(p, NT, info.sms, st);
            default: return launch_stream_cpt<N, S, KIND, 8>(p, NT, info.sms, st);
        }
    }
}

template <typename S, int KIND>
hc_status dispatch_n(int n, const hc::StepParams &p, cudaStream_t st) {
    switch (n) {
        case 1: return launch_stream<1, S, KIND>(p, st);
        case 2: return launch_stream<2, S, KIND>(p, st);
        case 3: return launch_stream<3, S, KIND>(p, st);
        case 4: return launch_stream<4, S, KIND>(p, st);
        case 5: return launch_stream<5, S, KIND>(p, st);
        case 6: return launch_stream<6, S, KIND>(p, st);
        case 7: return launch_stream<7, S, KIND>(p, st);
        default: return launch_stream<8, S, KIND>(p, st);
    }
}

template <int KIND>
hc_status dispatch(hc_dtype dt, int n, const hc::StepParams &p, cudaStream_t st) {
    if (dt == HC_BF16) return dispatch_n<__nv_bfloat16, KIND>(n, p, st);
    return dispatch_n<float, KIND>(n, p, st);
}

}  // namespace

// ============================== C ABI ==========================================

extern "C" {

int hc_version(void) { return 100; }

const char *hc_status_string(hc_status st) {
    switch (st) {
        case HC_OK: return "ok";
        case HC_ERR_INVALID_ARG: return "invalid argument";
        case HC_ERR_UNSUPPORTED: return "unsupported shape or option";
        case HC_ERR_MISALIGNED: return "misaligned pointer";
        case HC_ERR_ALIAS: return "output overlaps another buffer";
        case HC_ERR_CUDA: return "CUDA runtime error";
        case HC_ERR_DEVICE: return "device-side failure";
    }
    return "unknown status";
}

const char *hc_last_error(void) { return g_last_error; }

hc_status hc_sinkhorn(const float *logits, float *out, int64_t T, int n, int K, hc_stream stream) {
    static const char *fn = "hc_sinkhorn";
    g_last_error[0] = '\0';
    if (T < 0) return fail(HC_ERR_INVALID_ARG, "%s: T < 0", fn);
    if (n < 1) return fail(HC_ERR_INVALID_ARG, "%s: n = %d < 1", fn, n);
    if (n > hc::kMaxStreams) return fail(HC_ERR_UNSUPPORTED, "%s: n = %d > 8", fn, n);
    HC_TRY(check_K(fn, K));
    if (T == 0) return HC_OK;
    HC_TRY(check_param(fn, "logits", logits));
    HC_TRY(check_param(fn, "out", out));
    const int64_t bytes = T * n * n * 4;
    if (out != logits && overlap(out, bytes, logits, bytes))
        return fail(HC_ERR_ALIAS, "%s: out partially overlaps logits", fn);
    DeviceInfo info;
    HC_TRY(device_info(info));
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    const int threads = 256;
    int tpw = 1;
    switch (n) {
        case 1: tpw = hc::Group<1>::TPW; break;
        case 2: tpw = hc::Group<2>::TPW; break;
        case 3: tpw = hc::Group<3>::TPW; break;
        case 4: tpw = hc::Group<4>::TPW; break;
        default: tpw = 1; break;
    }
    const int64_t tokens_per_cta = (int64_t)(threads / 32) * tpw;
    int64_t grid = (T + tokens_per_cta - 1) / tokens_per_cta;
    const int64_t gmax = (int64_t)info.sms * 8;
    if (grid > gmax) grid = gmax;
    switch (n) {
        case 1: hc::hc_sinkhorn_kernel<1><<<(unsigned)grid, threads, 0, st>>>(logits, out, T, K); break;
        case 2: hc::hc_sinkhorn_kernel<2><<<(unsigned)grid, threads, 0, st>>>(logits, out, T, K); break;
        case 3: hc::hc_sinkhorn_kernel<3><<<(unsigned)grid, threads, 0, st>>>(logits, out, T, K); break;
        case 4: hc::hc_sinkhorn_kernel<4><<<(unsigned)grid, threads, 0, st>>>(logits, out, T, K); break;
        case 5: hc::hc_sinkhorn_kernel<5><<<(unsigned)grid, threads, 0, st>>>(logits, out, T, K); break;
        case 6: hc::hc_sinkhorn_kernel<6><<<(unsigned)grid, threads, 0, st>>>(logits, out, T, K); break;
        case 7: hc::hc_sinkhorn_kernel<7><<<(unsigned)grid, threads, 0, st>>>(logits, out, T, K); break;
        default: hc::hc_sinkhorn_kernel<8><<<(unsigned)grid, threads, 0, st>>>(logits, out, T, K); break;
    }
    return check_launch(fn);
}

hc_status hc_read_rmsnorm(const void *H, void *x, hc_dtype dt, int64_t T, int n, int64_t d,
                          hc_read_mode rm, const float *a, int64_t a_tok_stride, const float *g,
                          float eps, hc_stream stream) {
    static const char *fn = "hc_read_rmsnorm";
    g_last_error[0] = '\0';
    const Shape s{dt, T, n, d};
    HC_TRY(check_shape(fn, s, true));
    if (rm != HC_READ_WEIGHTS && rm != HC_READ_SOFTMAX_LOGITS)
        return fail(HC_ERR_INVALID_ARG, "%s: bad read mode %d", fn, (int)rm);
    HC_TRY(check_stride(fn, "a_tok_stride", a_tok_stride));
    HC_TRY(check_eps(fn, eps));
    if (T == 0) return HC_OK;
    HC_TRY(check_buf(fn, "H", H));
    HC_TRY(check_buf(fn, "x", x));
    HC_TRY(check_param(fn, "a", a));
    if (g && !aligned(g, 16)) return fail(HC_ERR_MISALIGNED, "%s: g is not 16-byte aligned", fn);
    const int64_t es = elem_bytes(dt);
    if (overlap(x, T * d * es, H, T * n * d * es)) return fail(HC_ERR_ALIAS, "%s: x overlaps H", fn);
    hc::StepParams p{};
    p.H = H; p.x = x; p.T = T; p.d = d;
    p.a = a; p.a_s = a_tok_stride; p.g = g; p.eps = eps;
    p.read_logits = rm == HC_READ_SOFTMAX_LOGITS;
    return dispatch<hc::KIND_READ>(dt, n, p, static_cast<cudaStream_t>(stream));
}

hc_status hc_write_mix(const void *H, const void *y, void *Hout, hc_dtype dt, int64_t T, int n,
                       int64_t d, hc_mix_mode mm, const float *A, int64_t A_tok_stride, int K,
                       const float *b, int64_t b_tok_stride, hc_stream stream) {
    static const char *fn = "hc_write_mix";
    g_last_error[0] = '\0';
    const Shape s{dt, T, n, d};
    HC_TRY(check_shape(fn, s, false));
    if (mm != HC_MIX_MATRIX && mm != HC_MIX_SINKHORN_LOGITS)
        return fail(HC_ERR_INVALID_ARG, "%s: bad mix mode %d", fn, (int)mm);
    if (mm == HC_MIX_SINKHORN_LOGITS) HC_TRY(check_K(fn, K));
    HC_TRY(check_stride(fn, "A_tok_stride", A_tok_stride));
    HC_TRY(check_stride(fn, "b_tok_stride", b_tok_stride));
    if (T == 0) return HC_OK;
    HC_TRY(check_buf(fn, "H", H));
    HC_TRY(check_buf(fn, "y", y));
    HC_TRY(check_buf(fn, "Hout", Hout));
    HC_TRY(check_param(fn, "A", A));
    HC_TRY(check_param(fn, "b", b));
    const int64_t es = elem_bytes(dt);
    const int64_t hb = T * n * d * es, yb = T * d * es;
    if (Hout != H && overlap(Hout, hb, H, hb)) return fail(HC_ERR_ALIAS, "%s: Hout partially overlaps H", fn);
    if (overlap(Hout, hb, y, yb)) return fail(HC_ERR_ALIAS, "%s: Hout overlaps y", fn);
    hc::StepParams p{};
    p.H = H; p.y = y; p.Hout = Hout; p.T = T; p.d = d;
    p.A = A; p.A_s = A_tok_stride; p.b = b; p.b_s = b_tok_stride;
    p.K = K; p.mix_logits = mm == HC_MIX_SINKHORN_LOGITS;
    return dispatch<hc::KIND_WRITE>(dt, n, p, static_cast<cudaStream_t>(stream));
}

hc_status hc_write_then_read(const void *H, const void *y, void *Hout, void *x_next, hc_dtype dt,
                             int64_t T, int n, int64_t d, hc_mix_mode mm, const float *A,
                             int64_t A_tok_stride, int K, const float *b, int64_t b_tok_stride,
                             hc_read_mode rm, const float *a_next, int64_t a_tok_stride,
                             const float *g_next, float eps, hc_stream stream) {
    static const char *fn = "hc_write_then_read";
    g_last_error[0] = '\0';
    const Shape s{dt, T, n, d};
    HC_TRY(check_shape(fn, s, true));
    if (mm != HC_MIX_MATRIX && mm != HC_MIX_SINKHORN_LOGITS)
        return fail(HC_ERR_INVALID_ARG, "%s: bad mix mode %d", fn, (int)mm);
    if (rm != HC_READ_WEIGHTS && rm != HC_READ_SOFTMAX_LOGITS)
        return fail(HC_ERR_INVALID_ARG, "%s: bad read mode %d", fn, (int)rm);
    if (mm == HC_MIX_SINKHORN_LOGITS) HC_TRY(check_K(fn, K));
    HC_TRY(check_stride(fn, "A_tok_stride", A_tok_stride));
    HC_TRY(check_stride(fn, "b_tok_stride", b_tok_stride));
    HC_TRY(check_stride(fn, "a_tok_stride", a_tok_stride));
    HC_TRY(check_eps(fn, eps));
    if (T == 0) return HC_OK;
    HC_TRY(check_buf(fn, "H", H));
    HC_TRY(check_buf(fn, "y", y));
    HC_TRY(check_buf(fn, "Hout", Hout));
    HC_TRY(check_buf(fn, "x_next", x_next));
    HC_TRY(check_param(fn, "A", A));
    HC_TRY(check_param(fn, "b", b));
    HC_TRY(check_param(fn, "a_next", a_next));
    if (g_next && !aligned(g_next, 16))
        return fail(HC_ERR_MISALIGNED, "%s: g_next is not 16-byte aligned", fn);
    const int64_t es = elem_bytes(dt);
    const int64_t hb = T * n * d * es, yb = T * d * es;
    if (Hout != H && overlap(Hout, hb, H, hb)) return fail(HC_ERR_ALIAS, "%s: Hout partially overlaps H", fn);
    if (overlap(Hout, hb, y, yb)) return fail(HC_ERR_ALIAS, "%s: Hout overlaps y", fn);
    if (overlap(x_next, yb, H, hb) || overlap(x_next, yb, Hout, hb) || overlap(x_next, yb, y, yb))
        return fail(HC_ERR_ALIAS, "%s: x_next overlaps H, Hout or y", fn);
    hc::StepParams p{};
    p.H = H; p.y = y; p.Hout = Hout; p.x = x_next; p.T = T; p.d = d;
    p.A = A; p.A_s = A_tok_stride; p.b = b; p.b_s = b_tok_stride;
    p.a = a_next; p.a_s = a_tok_stride; p.g = g_next; p.eps = eps;
    p.K = K; p.mix_logits = mm == HC_MIX_SINKHORN_LOGITS;
    p.read_logits = rm == HC_READ_SOFTMAX_LOGITS;
    return dispatch<hc::KIND_FUSED>(dt, n, p, static_cast<cudaStream_t>(stream));
}

}  // extern "C"
