// hc_api.cu -- host side of libhc_b200.so: argument validation, launch
// configuration and error reporting for the HC step kernels (the C ABI is
// declared in include/hc_api.h).
//
// Nothing here allocates device memory or synchronises; every launch goes on
// the caller's stream.

#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include <climits>
#include <cmath>
#include <cstdarg>
#include <cstdio>
#include <cstring>

#include <atomic>

#include "hc_api.h"
#include "hc_launch.h"

// The library's device fault word (one per device that loads the library).
// Pipelined kernels OR a fault code into it when a bounded wait runs out.
__device__ int g_hc_device_fault = 0;

namespace hc {

namespace {
thread_local char g_last_error[512] = "";
std::atomic<int> g_path{0};
}  // namespace

hc_status set_error(hc_status st, const char *fmt, ...) {
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(g_last_error, sizeof g_last_error, fmt, ap);
    va_end(ap);
    return st;
}

}  // namespace hc

namespace {

using hc::g_last_error;
#define fail hc::set_error

bool aligned(const void *p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

bool overlap(const void *p, int64_t pb, const void *q, int64_t qb) {
    if (!p || !q || pb <= 0 || qb <= 0) return false;
    const uintptr_t a0 = reinterpret_cast<uintptr_t>(p), a1 = a0 + (uintptr_t)pb;
    const uintptr_t b0 = reinterpret_cast<uintptr_t>(q), b1 = b0 + (uintptr_t)qb;
    return a0 < b1 && b0 < a1;
}

int elem_bytes(hc_dtype dt) { return dt == HC_BF16 ? 2 : 4; }
int vec_elems(hc_dtype dt) { return dt == HC_BF16 ? 8 : 4; }

// Per-device launch context: SM count and the address of this device's fault
// word (looked up once per device, with that device current).
hc_status launch_ctx(hc::LaunchCtx &ctx) {
    // published with release/acquire: the SM count is stored last and read first
    static std::atomic<int> sms_cache[64];
    static std::atomic<int *> fault_cache[64];
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return fail(HC_ERR_CUDA, "cudaGetDevice: %s", cudaGetErrorString(e));
    if (dev < 0 || dev >= 64) return fail(HC_ERR_UNSUPPORTED, "device ordinal %d >= 64", dev);
    int sms_known = sms_cache[dev].load(std::memory_order_acquire);
    if (sms_known == 0) {
        int sms = 0;
        e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
        if (e != cudaSuccess)
            return fail(HC_ERR_CUDA, "cudaDeviceGetAttribute: %s", cudaGetErrorString(e));
        void *addr = nullptr;
        e = cudaGetSymbolAddress(&addr, g_hc_device_fault);
        if (e != cudaSuccess)
            return fail(HC_ERR_CUDA, "cudaGetSymbolAddress(fault word): %s", cudaGetErrorString(e));
        fault_cache[dev].store(static_cast<int *>(addr), std::memory_order_relaxed);
        sms_cache[dev].store(sms, std::memory_order_release);
        sms_known = sms;
    }
    ctx.device = dev;
    ctx.sms = sms_known;
    ctx.fault = fault_cache[dev].load(std::memory_order_relaxed);
    ctx.path = hc::g_path.load(std::memory_order_relaxed);
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

template <int KIND>
hc_status dispatch(hc_dtype dt, int n, const hc::StepParams &p, cudaStream_t st) {
    hc::LaunchCtx ctx{};
    HC_TRY(launch_ctx(ctx));
    if (dt == HC_BF16) return hc::launch_kind<__nv_bfloat16, KIND>(n, p, ctx, st);
    return hc::launch_kind<float, KIND>(n, p, ctx, st);
}

}  // namespace

// ============================== C ABI ==========================================

extern "C" {

int hc_version(void) { return 300; }

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

hc_status hc_set_path(hc_path path) {
    g_last_error[0] = '\0';
    if (path != HC_PATH_AUTO && path != HC_PATH_PIPELINED && path != HC_PATH_REGISTER)
        return fail(HC_ERR_INVALID_ARG, "hc_set_path: bad path %d", (int)path);
    hc::g_path.store((int)path, std::memory_order_relaxed);
    return HC_OK;
}

hc_path hc_get_path(void) { return (hc_path)hc::g_path.load(std::memory_order_relaxed); }

hc_status hc_step_path(hc_dtype dt, int op, int64_t T, int n, int64_t d, hc_path *path) {
    static const char *fn = "hc_step_path";
    g_last_error[0] = '\0';
    if (!path) return fail(HC_ERR_INVALID_ARG, "%s: path is NULL", fn);
    if (op < 0 || op > 2) return fail(HC_ERR_INVALID_ARG, "%s: bad op %d", fn, op);
    const Shape s{dt, T, n, d};
    HC_TRY(check_shape(fn, s, op != 1));
    if (T < 1) return fail(HC_ERR_INVALID_ARG, "%s: T = %lld < 1", fn, (long long)T);
    hc::LaunchCtx ctx{};
    HC_TRY(launch_ctx(ctx));
    hc::StepParams p{};
    p.T = T;
    p.d = d;
    int r;
    if (dt == HC_BF16)
        r = op == 0   ? hc::step_path<__nv_bfloat16, hc::KIND_READ>(n, p, ctx)
            : op == 1 ? hc::step_path<__nv_bfloat16, hc::KIND_WRITE>(n, p, ctx)
                      : hc::step_path<__nv_bfloat16, hc::KIND_FUSED>(n, p, ctx);
    else
        r = op == 0   ? hc::step_path<float, hc::KIND_READ>(n, p, ctx)
            : op == 1 ? hc::step_path<float, hc::KIND_WRITE>(n, p, ctx)
                      : hc::step_path<float, hc::KIND_FUSED>(n, p, ctx);
    *path = (hc_path)r;
    return HC_OK;
}

hc_status hc_device_fault(int *code, hc_stream stream) {
    g_last_error[0] = '\0';
    if (!code) return fail(HC_ERR_INVALID_ARG, "hc_device_fault: code is NULL");
    hc::LaunchCtx ctx{};
    HC_TRY(launch_ctx(ctx));
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    cudaError_t e = cudaStreamSynchronize(st);
    if (e != cudaSuccess) return fail(HC_ERR_CUDA, "hc_device_fault: %s", cudaGetErrorString(e));
    int v = 0;
    e = cudaMemcpy(&v, ctx.fault, sizeof v, cudaMemcpyDeviceToHost);
    if (e == cudaSuccess && v != 0) e = cudaMemset(ctx.fault, 0, sizeof v);
    if (e != cudaSuccess) return fail(HC_ERR_CUDA, "hc_device_fault: %s", cudaGetErrorString(e));
    *code = v;
    return v ? fail(HC_ERR_DEVICE, "device fault code 0x%x", v) : HC_OK;
}

hc_status hc_mix_logits(const void *H, const void *W, float *logits, hc_dtype dt, int64_t T, int n,
                        int64_t d, int P, float eps, hc_stream stream) {
    static const char *fn = "hc_mix_logits";
    g_last_error[0] = '\0';
    const Shape s{dt, T, n, d};
    HC_TRY(check_shape(fn, s, false));
    if (dt != HC_BF16) return fail(HC_ERR_UNSUPPORTED, "%s: only bf16 streams and weights", fn);
    if (P < 1) return fail(HC_ERR_INVALID_ARG, "%s: P = %d < 1", fn, P);
    if (P > 256) return fail(HC_ERR_UNSUPPORTED, "%s: P = %d > 256", fn, P);
    HC_TRY(check_eps(fn, eps));
    // TMA coordinates are 32-bit and run up to one tile past the end
    if (T > (int64_t)0x7fffff00 || (int64_t)n * d > (int64_t)0x7fffff00)
        return fail(HC_ERR_UNSUPPORTED, "%s: T or n*d beyond 2^31 - 256", fn);
    if (T == 0) return HC_OK;
    HC_TRY(check_buf(fn, "H", H));
    HC_TRY(check_buf(fn, "W", W));
    HC_TRY(check_param(fn, "logits", logits));
    const int64_t hb = T * n * d * 2, wb = (int64_t)P * n * d * 2, zb = T * P * 4;
    if (overlap(logits, zb, H, hb) || overlap(logits, zb, W, wb))
        return fail(HC_ERR_ALIAS, "%s: logits overlap H or W", fn);
    hc::LaunchCtx ctx{};
    HC_TRY(launch_ctx(ctx));
    return hc::launch_mix_logits(H, W, logits, T, n, d, P, eps, ctx, static_cast<cudaStream_t>(stream));
}

hc_status hc_selftest_bounded_wait(int limit_us, hc_stream stream) {
    g_last_error[0] = '\0';
    if (limit_us < 1 || limit_us > 100000)
        return fail(HC_ERR_INVALID_ARG, "hc_selftest_bounded_wait: limit_us = %d not in [1, 100000]",
                    limit_us);
    hc::LaunchCtx ctx{};
    HC_TRY(launch_ctx(ctx));
    return hc::launch_selftest_wait(limit_us, ctx, static_cast<cudaStream_t>(stream));
}

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
    hc::LaunchCtx ctx{};
    HC_TRY(launch_ctx(ctx));
    return hc::launch_sinkhorn(logits, out, T, n, K, ctx, static_cast<cudaStream_t>(stream));
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

hc_status hc_expand(const void *x, void *H, hc_dtype dt, int64_t T, int n, int64_t d,
                    hc_stream stream) {
    static const char *fn = "hc_expand";
    g_last_error[0] = '\0';
    const Shape s{dt, T, n, d};
    HC_TRY(check_shape(fn, s, false));
    if (T == 0) return HC_OK;
    HC_TRY(check_buf(fn, "x", x));
    HC_TRY(check_buf(fn, "H", H));
    const int64_t es = elem_bytes(dt);
    if (overlap(H, T * n * d * es, x, T * d * es)) return fail(HC_ERR_ALIAS, "%s: H overlaps x", fn);
    hc::StepParams p{};
    p.y = x; p.Hout = H; p.T = T; p.d = d;
    return dispatch<hc::KIND_EXPAND>(dt, n, p, static_cast<cudaStream_t>(stream));
}

hc_status hc_expand_then_read(const void *x, void *H, void *x_read, hc_dtype dt, int64_t T, int n,
                              int64_t d, hc_read_mode rm, const float *a, int64_t a_tok_stride,
                              const float *g, float eps, hc_stream stream) {
    static const char *fn = "hc_expand_then_read";
    g_last_error[0] = '\0';
    const Shape s{dt, T, n, d};
    HC_TRY(check_shape(fn, s, true));
    if (rm != HC_READ_WEIGHTS && rm != HC_READ_SOFTMAX_LOGITS)
        return fail(HC_ERR_INVALID_ARG, "%s: bad read mode %d", fn, (int)rm);
    HC_TRY(check_stride(fn, "a_tok_stride", a_tok_stride));
    HC_TRY(check_eps(fn, eps));
    if (T == 0) return HC_OK;
    HC_TRY(check_buf(fn, "x", x));
    HC_TRY(check_buf(fn, "H", H));
    HC_TRY(check_buf(fn, "x_read", x_read));
    HC_TRY(check_param(fn, "a", a));
    if (g && !aligned(g, 16)) return fail(HC_ERR_MISALIGNED, "%s: g is not 16-byte aligned", fn);
    const int64_t es = elem_bytes(dt);
    const int64_t hb = T * n * d * es, xb = T * d * es;
    if (overlap(H, hb, x, xb)) return fail(HC_ERR_ALIAS, "%s: H overlaps x", fn);
    if (overlap(x_read, xb, H, hb)) return fail(HC_ERR_ALIAS, "%s: x_read overlaps H", fn);
    if (x_read != x && overlap(x_read, xb, x, xb))
        return fail(HC_ERR_ALIAS, "%s: x_read partially overlaps x", fn);
    hc::StepParams p{};
    p.y = x; p.Hout = H; p.x = x_read; p.T = T; p.d = d;
    p.a = a; p.a_s = a_tok_stride; p.g = g; p.eps = eps;
    p.read_logits = rm == HC_READ_SOFTMAX_LOGITS;
    return dispatch<hc::KIND_EXPAND_READ>(dt, n, p, static_cast<cudaStream_t>(stream));
}

hc_status hc_collapse(const void *H, void *out, hc_dtype dt, int64_t T, int n, int64_t d,
                      hc_read_mode rm, const float *w, int64_t w_tok_stride, hc_stream stream) {
    static const char *fn = "hc_collapse";
    g_last_error[0] = '\0';
    const Shape s{dt, T, n, d};
    HC_TRY(check_shape(fn, s, false));
    if (rm != HC_READ_WEIGHTS && rm != HC_READ_SOFTMAX_LOGITS)
        return fail(HC_ERR_INVALID_ARG, "%s: bad read mode %d", fn, (int)rm);
    HC_TRY(check_stride(fn, "w_tok_stride", w_tok_stride));
    if (T == 0) return HC_OK;
    HC_TRY(check_buf(fn, "H", H));
    HC_TRY(check_buf(fn, "out", out));
    HC_TRY(check_param(fn, "w", w));
    const int64_t es = elem_bytes(dt);
    if (overlap(out, T * d * es, H, T * n * d * es)) return fail(HC_ERR_ALIAS, "%s: out overlaps H", fn);
    hc::StepParams p{};
    p.H = H; p.x = out; p.T = T; p.d = d;
    p.a = w; p.a_s = w_tok_stride;
    p.read_logits = rm == HC_READ_SOFTMAX_LOGITS;
    return dispatch<hc::KIND_COLLAPSE>(dt, n, p, static_cast<cudaStream_t>(stream));
}

hc_status hc_reduce_write_then_read(const void *const *y_parts, int R, const void *H, void *Hout,
                                    void *x_next, void *y_out, hc_dtype dt, int64_t T, int n,
                                    int64_t d, hc_mix_mode mm, const float *A, int64_t A_tok_stride,
                                    int K, const float *b, int64_t b_tok_stride, hc_read_mode rm,
                                    const float *a_next, int64_t a_tok_stride, const float *g_next,
                                    float eps, hc_stream stream) {
    static const char *fn = "hc_reduce_write_then_read";
    g_last_error[0] = '\0';
    const Shape s{dt, T, n, d};
    HC_TRY(check_shape(fn, s, true));
    if (R < 1) return fail(HC_ERR_INVALID_ARG, "%s: R = %d < 1", fn, R);
    if (R > hc::kMaxRanks) return fail(HC_ERR_UNSUPPORTED, "%s: R = %d > %d", fn, R, hc::kMaxRanks);
    if (!y_parts) return fail(HC_ERR_INVALID_ARG, "%s: y_parts is NULL", fn);
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
    HC_TRY(check_buf(fn, "Hout", Hout));
    HC_TRY(check_buf(fn, "x_next", x_next));
    for (int r = 0; r < R; ++r) {
        char name[24];
        snprintf(name, sizeof name, "y_parts[%d]", r);
        HC_TRY(check_buf(fn, name, y_parts[r]));
    }
    if (y_out && !aligned(y_out, 16)) return fail(HC_ERR_MISALIGNED, "%s: y_out is not 16-byte aligned", fn);
    HC_TRY(check_param(fn, "A", A));
    HC_TRY(check_param(fn, "b", b));
    HC_TRY(check_param(fn, "a_next", a_next));
    if (g_next && !aligned(g_next, 16))
        return fail(HC_ERR_MISALIGNED, "%s: g_next is not 16-byte aligned", fn);
    const int64_t es = elem_bytes(dt);
    const int64_t hb = T * n * d * es, yb = T * d * es;
    if (Hout != H && overlap(Hout, hb, H, hb)) return fail(HC_ERR_ALIAS, "%s: Hout partially overlaps H", fn);
    if (overlap(x_next, yb, H, hb) || overlap(x_next, yb, Hout, hb))
        return fail(HC_ERR_ALIAS, "%s: x_next overlaps H or Hout", fn);
    if (y_out && (overlap(y_out, yb, H, hb) || overlap(y_out, yb, Hout, hb) || overlap(y_out, yb, x_next, yb)))
        return fail(HC_ERR_ALIAS, "%s: y_out overlaps H, Hout or x_next", fn);
    for (int r = 0; r < R; ++r) {
        const void *q = y_parts[r];
        if (overlap(Hout, hb, q, yb) || overlap(x_next, yb, q, yb) || (y_out && overlap(y_out, yb, q, yb)))
            return fail(HC_ERR_ALIAS, "%s: an output overlaps y_parts[%d]", fn, r);
    }
    hc::LaunchCtx ctx{};
    HC_TRY(launch_ctx(ctx));
    hc::ReduceWriteArgs ra{};
    ra.f.H = H; ra.f.Hout = Hout; ra.f.T = T; ra.f.d = d;
    ra.f.A = A; ra.f.A_s = A_tok_stride; ra.f.b = b; ra.f.b_s = b_tok_stride;
    ra.f.a = a_next; ra.f.a_s = a_tok_stride; ra.f.g = g_next; ra.f.eps = eps;
    ra.f.K = K; ra.f.mix_logits = mm == HC_MIX_SINKHORN_LOGITS;
    ra.f.read_logits = rm == HC_READ_SOFTMAX_LOGITS;
    for (int r = 0; r < R; ++r) ra.parts[r] = y_parts[r];
    ra.R = R;
    ra.n = n;
    ra.y_out = y_out;
    ra.t0 = 0;
    ra.xs[0] = x_next;
    ra.nx = 1;
    return hc::launch_reduce_write(ra, dt, ctx, static_cast<cudaStream_t>(stream));
}

hc_status hc_reduce_scatter_write_then_read(const void *const *y_parts, int R, int rank,
                                            int64_t T_total, const void *H, void *Hout,
                                            void *const *x_all, void *y_out, hc_dtype dt, int n,
                                            int64_t d, hc_mix_mode mm, const float *A,
                                            int64_t A_tok_stride, int K, const float *b,
                                            int64_t b_tok_stride, hc_read_mode rm,
                                            const float *a_next, int64_t a_tok_stride,
                                            const float *g_next, float eps, hc_stream stream) {
    static const char *fn = "hc_reduce_scatter_write_then_read";
    g_last_error[0] = '\0';
    if (R < 1) return fail(HC_ERR_INVALID_ARG, "%s: R = %d < 1", fn, R);
    if (R > hc::kMaxRanks) return fail(HC_ERR_UNSUPPORTED, "%s: R = %d > %d", fn, R, hc::kMaxRanks);
    if (rank < 0 || rank >= R) return fail(HC_ERR_INVALID_ARG, "%s: rank %d outside 0..%d", fn, rank, R - 1);
    HC_TRY(check_shape(fn, Shape{dt, T_total, n, d}, true));
    // this rank's tokens: contiguous shards, the first T_total % R one longer
    const int64_t base = T_total / R, extra = T_total % R;
    const int64_t t0 = rank * base + (rank < extra ? rank : extra);
    const int64_t T = base + (rank < extra ? 1 : 0);
    if (!y_parts) return fail(HC_ERR_INVALID_ARG, "%s: y_parts is NULL", fn);
    if (!x_all) return fail(HC_ERR_INVALID_ARG, "%s: x_all is NULL", fn);
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
    HC_TRY(check_buf(fn, "Hout", Hout));
    for (int r = 0; r < R; ++r) {
        char name[24];
        snprintf(name, sizeof name, "y_parts[%d]", r);
        HC_TRY(check_buf(fn, name, y_parts[r]));
        snprintf(name, sizeof name, "x_all[%d]", r);
        HC_TRY(check_buf(fn, name, x_all[r]));
    }
    if (y_out && !aligned(y_out, 16)) return fail(HC_ERR_MISALIGNED, "%s: y_out is not 16-byte aligned", fn);
    HC_TRY(check_param(fn, "A", A));
    HC_TRY(check_param(fn, "b", b));
    HC_TRY(check_param(fn, "a_next", a_next));
    if (g_next && !aligned(g_next, 16))
        return fail(HC_ERR_MISALIGNED, "%s: g_next is not 16-byte aligned", fn);
    const int64_t es = elem_bytes(dt);
    const int64_t hb = T * n * d * es, yb = T * d * es, fb = T_total * d * es;
    if (Hout != H && overlap(Hout, hb, H, hb)) return fail(HC_ERR_ALIAS, "%s: Hout partially overlaps H", fn);
    if (y_out && (overlap(y_out, yb, H, hb) || overlap(y_out, yb, Hout, hb)))
        return fail(HC_ERR_ALIAS, "%s: y_out overlaps H or Hout", fn);
    for (int q = 0; q < R; ++q) {
        const void *xq = x_all[q], *pq = y_parts[q];
        if (overlap(xq, fb, H, hb) || overlap(xq, fb, Hout, hb) || (y_out && overlap(xq, fb, y_out, yb)))
            return fail(HC_ERR_ALIAS, "%s: x_all[%d] overlaps H, Hout or y_out", fn, q);
        if (overlap(Hout, hb, pq, fb) || (y_out && overlap(y_out, yb, pq, fb)))
            return fail(HC_ERR_ALIAS, "%s: an output overlaps y_parts[%d]", fn, q);
        for (int r = 0; r < R; ++r) {
            if (overlap(xq, fb, y_parts[r], fb))
                return fail(HC_ERR_ALIAS, "%s: x_all[%d] overlaps y_parts[%d]", fn, q, r);
            if (r > q && overlap(xq, fb, x_all[r], fb))
                return fail(HC_ERR_ALIAS, "%s: x_all[%d] overlaps x_all[%d]", fn, q, r);
        }
    }
    hc::LaunchCtx ctx{};
    HC_TRY(launch_ctx(ctx));
    hc::ReduceWriteArgs ra{};
    ra.f.H = H; ra.f.Hout = Hout; ra.f.T = T; ra.f.d = d;
    ra.f.A = A; ra.f.A_s = A_tok_stride; ra.f.b = b; ra.f.b_s = b_tok_stride;
    ra.f.a = a_next; ra.f.a_s = a_tok_stride; ra.f.g = g_next; ra.f.eps = eps;
    ra.f.K = K; ra.f.mix_logits = mm == HC_MIX_SINKHORN_LOGITS;
    ra.f.read_logits = rm == HC_READ_SOFTMAX_LOGITS;
    for (int r = 0; r < R; ++r) {
        ra.parts[r] = y_parts[r];
        ra.xs[r] = x_all[r];
    }
    ra.R = R;
    ra.nx = R;
    ra.n = n;
    ra.y_out = y_out;
    ra.t0 = t0;
    return hc::launch_reduce_write(ra, dt, ctx, static_cast<cudaStream_t>(stream));
}

hc_status hc_ipc_export(const void *dev_ptr, void *handle, uint64_t *offset) {
    static const char *fn = "hc_ipc_export";
    g_last_error[0] = '\0';
    if (!dev_ptr || !handle || !offset) return fail(HC_ERR_INVALID_ARG, "%s: NULL argument", fn);
    // looked up once (thread-safe static initialisation); null if unavailable
    static const PFN_cuMemGetAddressRange_v3020 range_fn = [] {
        void *fp = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuMemGetAddressRange", &fp, cudaEnableDefault, &q) != cudaSuccess ||
            q != cudaDriverEntryPointSuccess)
            fp = nullptr;
        return reinterpret_cast<PFN_cuMemGetAddressRange_v3020>(fp);
    }();
    if (!range_fn) return fail(HC_ERR_CUDA, "%s: cuMemGetAddressRange is not available", fn);
    CUdeviceptr base = 0;
    size_t bytes = 0;
    const CUresult cr = range_fn(&base, &bytes, reinterpret_cast<CUdeviceptr>(dev_ptr));
    if (cr != CUDA_SUCCESS) return fail(HC_ERR_CUDA, "%s: cuMemGetAddressRange failed (%d)", fn, (int)cr);
    cudaIpcMemHandle_t h;
    const cudaError_t e = cudaIpcGetMemHandle(&h, reinterpret_cast<void *>(base));
    if (e != cudaSuccess) return fail(HC_ERR_CUDA, "%s: cudaIpcGetMemHandle: %s", fn, cudaGetErrorString(e));
    memcpy(handle, &h, sizeof h);
    *offset = (uint64_t)(reinterpret_cast<CUdeviceptr>(dev_ptr) - base);
    return HC_OK;
}

hc_status hc_ipc_open(const void *handle, void **base) {
    static const char *fn = "hc_ipc_open";
    g_last_error[0] = '\0';
    if (!handle || !base) return fail(HC_ERR_INVALID_ARG, "%s: NULL argument", fn);
    cudaIpcMemHandle_t h;
    memcpy(&h, handle, sizeof h);
    const cudaError_t e = cudaIpcOpenMemHandle(base, h, cudaIpcMemLazyEnablePeerAccess);
    if (e != cudaSuccess) return fail(HC_ERR_CUDA, "%s: cudaIpcOpenMemHandle: %s", fn, cudaGetErrorString(e));
    return HC_OK;
}

hc_status hc_ipc_close(void *base) {
    static const char *fn = "hc_ipc_close";
    g_last_error[0] = '\0';
    if (!base) return fail(HC_ERR_INVALID_ARG, "%s: base is NULL", fn);
    const cudaError_t e = cudaIpcCloseMemHandle(base);
    if (e != cudaSuccess) return fail(HC_ERR_CUDA, "%s: cudaIpcCloseMemHandle: %s", fn, cudaGetErrorString(e));
    return HC_OK;
}

hc_status hc_linear_then_write(const void *X, const void *Wo, const void *H, void *Hout, void *y_out,
                               hc_dtype dt, int64_t T, int n, int64_t d, int64_t k, const float *A,
                               int64_t A_tok_stride, const float *b, int64_t b_tok_stride,
                               hc_stream stream) {
    static const char *fn = "hc_linear_then_write";
    g_last_error[0] = '\0';
    if (dt != HC_BF16) return fail(HC_ERR_UNSUPPORTED, "%s: bf16 storage only (dtype %d)", fn, (int)dt);
    const Shape s{dt, T, n, d};
    HC_TRY(check_shape(fn, s, false));
    if (k < 1) return fail(HC_ERR_INVALID_ARG, "%s: k = %lld < 1", fn, (long long)k);
    if (k % 8 != 0)
        return fail(HC_ERR_UNSUPPORTED, "%s: k = %lld is not a multiple of 8 (16-byte rows)", fn,
                    (long long)k);
    // TMA coordinates are 32-bit and run up to one tile past the end
    const int64_t lim = (int64_t)0x7fffff00;
    if (k > lim || d > lim || T > lim)
        return fail(HC_ERR_UNSUPPORTED, "%s: T, d and k must each be below 2^31 - 256", fn);
    HC_TRY(check_stride(fn, "A_tok_stride", A_tok_stride));
    HC_TRY(check_stride(fn, "b_tok_stride", b_tok_stride));
    if (T == 0) return HC_OK;
    HC_TRY(check_buf(fn, "X", X));
    HC_TRY(check_buf(fn, "Wo", Wo));
    HC_TRY(check_buf(fn, "H", H));
    HC_TRY(check_buf(fn, "Hout", Hout));
    if (y_out && !aligned(y_out, 16)) return fail(HC_ERR_MISALIGNED, "%s: y_out is not 16-byte aligned", fn);
    HC_TRY(check_param(fn, "A", A));
    HC_TRY(check_param(fn, "b", b));
    const int64_t hb = T * n * d * 2, yb = T * d * 2, xb = T * k * 2, wb = d * k * 2;
    if (Hout != H && overlap(Hout, hb, H, hb)) return fail(HC_ERR_ALIAS, "%s: Hout partially overlaps H", fn);
    if (overlap(Hout, hb, X, xb) || overlap(Hout, hb, Wo, wb))
        return fail(HC_ERR_ALIAS, "%s: Hout overlaps X or Wo", fn);
    if (y_out && (overlap(y_out, yb, H, hb) || overlap(y_out, yb, Hout, hb) ||
                  overlap(y_out, yb, X, xb) || overlap(y_out, yb, Wo, wb)))
        return fail(HC_ERR_ALIAS, "%s: y_out overlaps another buffer", fn);
    hc::LaunchCtx ctx{};
    HC_TRY(launch_ctx(ctx));
    hc::LinearWriteArgs la{};
    la.X = X; la.Wo = Wo; la.H = H; la.Hout = Hout; la.y = y_out;
    la.T = T; la.d = d; la.k = k; la.n = n;
    la.A = A; la.A_s = A_tok_stride; la.b = b; la.b_s = b_tok_stride;
    return hc::launch_linear_write(la, ctx, static_cast<cudaStream_t>(stream));
}

size_t hc_write_then_read_backward_workspace_bytes(hc_dtype dt, int64_t T, int n, int64_t d) {
    if ((dt != HC_F32 && dt != HC_BF16) || T < 1 || n < 1 || n > hc::kMaxStreams || d < 1) return 0;
    hc::LaunchCtx ctx{};
    if (launch_ctx(ctx) != HC_OK) return 0;
    size_t bytes = 0;
    if (hc::backward_workspace_bytes(n, dt, T, d, ctx, &bytes) != HC_OK) return 0;
    return bytes;
}

hc_status hc_write_then_read_backward(const void *H, const void *y, hc_dtype dt, int64_t T, int n,
                                      int64_t d, hc_mix_mode mm, const float *A, int64_t A_tok_stride,
                                      int K, const float *b, int64_t b_tok_stride, hc_read_mode rm,
                                      const float *a, int64_t a_tok_stride, const float *g, float eps,
                                      const void *dHout, const void *dx, void *dH, void *dy,
                                      float *dA, float *db, float *da, float *dg, void *workspace,
                                      size_t workspace_bytes, hc_stream stream) {
    static const char *fn = "hc_write_then_read_backward";
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
    HC_TRY(check_buf(fn, "dx", dx));
    HC_TRY(check_buf(fn, "dH", dH));
    HC_TRY(check_buf(fn, "dy", dy));
    if (dHout && !aligned(dHout, 16)) return fail(HC_ERR_MISALIGNED, "%s: dHout is not 16-byte aligned", fn);
    HC_TRY(check_param(fn, "A", A));
    HC_TRY(check_param(fn, "b", b));
    HC_TRY(check_param(fn, "a", a));
    HC_TRY(check_param(fn, "dA", dA));
    HC_TRY(check_param(fn, "db", db));
    HC_TRY(check_param(fn, "da", da));
    if (g && !aligned(g, 16)) return fail(HC_ERR_MISALIGNED, "%s: g is not 16-byte aligned", fn);
    if (dg) {
        if (!g) return fail(HC_ERR_INVALID_ARG, "%s: dg requested without a gain g", fn);
        if (!aligned(dg, 4)) return fail(HC_ERR_MISALIGNED, "%s: dg is not 4-byte aligned", fn);
        if (!workspace) return fail(HC_ERR_INVALID_ARG, "%s: dg needs a workspace", fn);
        if (!aligned(workspace, 16)) return fail(HC_ERR_MISALIGNED, "%s: workspace is not 16-byte aligned", fn);
    }
    const int64_t es = elem_bytes(dt);
    const int64_t hb = T * n * d * es, yb = T * d * es;
    struct Span { const void *p; int64_t bytes; };
    const Span ins[] = {{H, hb}, {y, yb}, {dx, yb}, {dHout, dHout ? hb : 0}, {A, 0}, {b, 0}, {a, 0}, {g, 0}};
    const Span outs[] = {{dH, hb}, {dy, yb}, {dA, T * n * n * 4}, {db, T * n * 4}, {da, T * n * 4},
                         {dg, dg ? d * 4 : 0}, {workspace, dg ? (int64_t)workspace_bytes : 0}};
    for (const Span &o : outs) {
        if (!o.p || o.bytes == 0) continue;
        for (const Span &i : ins)
            if (i.p && i.bytes && overlap(o.p, o.bytes, i.p, i.bytes))
                return fail(HC_ERR_ALIAS, "%s: an output overlaps an input", fn);
        for (const Span &o2 : outs)
            if (&o2 != &o && o2.p && o2.bytes && overlap(o.p, o.bytes, o2.p, o2.bytes))
                return fail(HC_ERR_ALIAS, "%s: two outputs overlap", fn);
    }
    hc::LaunchCtx ctx{};
    HC_TRY(launch_ctx(ctx));
    hc::BackwardArgs ba{};
    ba.f.H = H; ba.f.y = y; ba.f.T = T; ba.f.d = d;
    ba.f.A = A; ba.f.A_s = A_tok_stride; ba.f.b = b; ba.f.b_s = b_tok_stride;
    ba.f.a = a; ba.f.a_s = a_tok_stride; ba.f.g = g; ba.f.eps = eps;
    ba.f.K = K; ba.f.mix_logits = mm == HC_MIX_SINKHORN_LOGITS;
    ba.f.read_logits = rm == HC_READ_SOFTMAX_LOGITS;
    ba.n = n; ba.dt = dt;
    ba.dHout = dHout; ba.dx = dx; ba.dH = dH; ba.dy = dy;
    ba.dA = dA; ba.db = db; ba.da = da; ba.dg = dg;
    ba.workspace = workspace; ba.workspace_bytes = workspace_bytes;
    return hc::launch_backward(ba, ctx, static_cast<cudaStream_t>(stream));
}

}  // extern "C"
