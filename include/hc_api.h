/*
 * hc_api.h -- C ABI of libhc_b200.so: the Hyper-Connections residual step on
 * NVIDIA B200 (sm_100a).
 *
 * The method ("Hyper-connections (mHC)" glossary entry, hfviewer, definition
 * paragraph): the transformer's single residual stream x + f(x) is widened to
 * n parallel streams H[n][d] per token; learned matrices mix the streams
 * before the block runs (read) and after it (write); the mHC variant makes
 * the mixing doubly stochastic with a few Sinkhorn iterations. Hy4 uses n = 4
 * ("Tencent open-sources Hy4 Preview at 770B -- Identity Hyper-Connections",
 * learnaivisually, TL;DR), and the block normalises its input (pre-norm,
 * same page, Jargon).
 *
 * Equations (the pages print none; these are the readings this library
 * implements):
 *   read   x    = RMSNorm(h) * g,  h = sum_i a_i H_i,
 *                 RMSNorm(h) = h / sqrt(mean_k(h_k^2) + eps)
 *   write  H'_j = sum_i A[i][j] H_i + b_j * y      (row i = source stream)
 *   mHC    A    = Sinkhorn_K(exp(L)): K times divide each row by its sum,
 *                 then each column by its sum (exactly K pairs, no early exit)
 *          a    = softmax(l) over the n streams (per-token read logits)
 *
 * Arithmetic: fp32 accumulation. Each mix is a chain of correctly rounded
 * fp32 fused multiply-adds in stream order starting from -0.0f; the stored
 * results (H', x) are rounded once to the storage dtype (bf16: round to
 * nearest even). The RMSNorm statistic sum_k h_k^2 is accumulated in fp64,
 * r = (float)(1 / sqrt(ss / d + eps)), and x = (h * r) * g in fp32. The
 * read of the fused call uses the stored (rounded) H'.
 *
 * Layout (row-major, no padding): H, Hout [T][n][d] (a token's n rows are
 * contiguous); y, x [T][d]; fp32 parameters. Per-token parameters take a
 * token stride in elements: 0 = one set shared by every token (a per-layer
 * parameter), otherwise the distance between consecutive tokens' sets
 * (n*n for A or L, n for a, b or l when densely packed).
 *
 * Conventions, all entry points:
 *  - Every pointer is a DEVICE pointer on the current CUDA device, allocated
 *    and owned by the caller. The library allocates nothing, frees nothing
 *    and never synchronises; work is enqueued on `stream` (a cudaStream_t;
 *    NULL = the legacy default stream) and completes asynchronously.
 *  - Arguments are validated on the host before anything is launched; on any
 *    error nothing is launched and the status says why (hc_last_error() has
 *    the details for the calling thread).
 *  - T == 0 is a no-op that returns HC_OK once the scalar arguments are valid.
 *  - Supported: 1 <= n <= 8; d > 0 with d % 8 == 0 (bf16) or d % 4 == 0
 *    (fp32); d <= 32768 (bf16) or 16384 (fp32) for calls that normalise.
 *    H, y, Hout, x and g are 16-byte aligned; A, b, a are 4-byte aligned.
 *  - Hout == H (exact in-place update) is allowed. Any other overlap between
 *    an output and another buffer returns HC_ERR_ALIAS.
 *  - NaN and Inf inputs propagate per IEEE 754; they are not checked.
 */
#ifndef HC_API_H
#define HC_API_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define HC_API __attribute__((visibility("default")))
#else
#define HC_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    HC_OK = 0,
    HC_ERR_INVALID_ARG = 1, /* null pointer, negative size or stride, bad enum, K < 1, eps < 0 */
    HC_ERR_UNSUPPORTED = 2, /* valid math, outside this library's limits (n > 8, d % 8 ...) */
    HC_ERR_MISALIGNED = 3,  /* a pointer misses the alignment stated above */
    HC_ERR_ALIAS = 4,       /* an output overlaps another buffer (other than Hout == H) */
    HC_ERR_CUDA = 5,        /* the CUDA runtime reported an error at launch */
    HC_ERR_DEVICE = 6       /* a kernel reported a device-side failure */
} hc_status;

typedef enum { HC_F32 = 0, HC_BF16 = 1 } hc_dtype;

/* How the write mix gets A: given directly, or as logits L projected per
 * token by K Sinkhorn iterations (mHC). */
typedef enum { HC_MIX_MATRIX = 0, HC_MIX_SINKHORN_LOGITS = 1 } hc_mix_mode;

/* How the read gets a: given directly, or as logits turned into weights by a
 * softmax over the n streams (mHC). */
typedef enum { HC_READ_WEIGHTS = 0, HC_READ_SOFTMAX_LOGITS = 1 } hc_read_mode;

typedef void *hc_stream; /* cudaStream_t */

/*
 * Sinkhorn projection ("Hyper-connections (mHC)", definition paragraph: the
 * mixing is made doubly stochastic with a few Sinkhorn iterations).
 *   logits [T][n][n] fp32 in, out [T][n][n] fp32 out (may equal logits).
 *   out = K x (row normalisation, column normalisation) of exp(logits).
 *   Columns of out sum to 1 (the column pass is last); rows approach 1 as K
 *   grows. 1 <= n <= 8, K >= 1. Both pointers 4-byte aligned, 16-byte not
 *   needed. A standalone entry for tests and for callers that keep A.
 */
HC_API hc_status hc_sinkhorn(const float *logits, float *out, int64_t T, int n, int K,
                      hc_stream stream);

/*
 * Read mix followed by the block's pre-norm RMSNorm ("Hyper-connections
 * (mHC)": mixing before the block; Hy4 explainer, Jargon "Pre-norm").
 *   H [T][n][d] in (dtype dt), x [T][d] out (dtype dt).
 *   rm == HC_READ_WEIGHTS: a holds weights; HC_READ_SOFTMAX_LOGITS: logits.
 *   a_tok_stride: 0 = one set of n for all tokens, else floats per token.
 *   g: [d] fp32 per-channel gain, or NULL for a gain of 1.
 *   eps >= 0, added to the mean square inside the square root.
 */
HC_API hc_status hc_read_rmsnorm(const void *H, void *x, hc_dtype dt, int64_t T, int n, int64_t d,
                          hc_read_mode rm, const float *a, int64_t a_tok_stride,
                          const float *g, float eps, hc_stream stream);

/*
 * Write mix ("Hyper-connections (mHC)": mixing after the block; Hy4 explainer,
 * TL;DR: a block can write to one stream and leave the others intact).
 *   H [T][n][d] and y [T][d] in, Hout [T][n][d] out, all dtype dt.
 *   H'_j = sum_i A[i][j] H_i + b_j y.
 *   mm == HC_MIX_MATRIX: A holds the n x n matrix (row-major, row = source);
 *   HC_MIX_SINKHORN_LOGITS: A holds logits and K >= 1 Sinkhorn pairs project
 *   them per token in registers (the matrix never goes to memory).
 *   A_tok_stride / b_tok_stride: 0 = shared by all tokens, else floats per token.
 *   Hout may equal H.
 */
HC_API hc_status hc_write_mix(const void *H, const void *y, void *Hout, hc_dtype dt, int64_t T, int n,
                       int64_t d, hc_mix_mode mm, const float *A, int64_t A_tok_stride, int K,
                       const float *b, int64_t b_tok_stride, hc_stream stream);

/*
 * Fused step: layer l's write followed by layer l+1's read + RMSNorm in one
 * pass over HBM, so H' is not read back. Same arguments as the two calls
 * above; the read uses the stored (rounded) H'. Hout may equal H; x_next must
 * not overlap H, Hout or y.
 */
HC_API hc_status hc_write_then_read(const void *H, const void *y, void *Hout, void *x_next,
                             hc_dtype dt, int64_t T, int n, int64_t d, hc_mix_mode mm,
                             const float *A, int64_t A_tok_stride, int K, const float *b,
                             int64_t b_tok_stride, hc_read_mode rm, const float *a_next,
                             int64_t a_tok_stride, const float *g_next, float eps,
                             hc_stream stream);

/*
 * The block's output projection fused with the write mix, so the block output
 * y never makes a round trip through HBM (Hy4-preview model techniques map,
 * models.inteligile.com, the "inference kernel" row, which records that Hy4's
 * kernels are fused; glossary entry "Hyper-connections (mHC)": the streams are
 * mixed after each block):
 *   y[t][c]  = bf16( sum_k X[t][k] * Wo[c][k] )   fp32 accumulation on the tensor
 *              cores, rounded to bf16 as a stored y would be;
 *   H'[t][j] = sum_i A[i][j] H[t][i] + b_j y[t]   as hc_write_mix with a given
 *              matrix (the per-token Sinkhorn form projects its logits first
 *              with hc_sinkhorn).
 *   X [T][k], Wo [d][k] (the projection's weight, one row per output channel),
 *   H and Hout [T][n][d]; bf16 only. k % 8 == 0, d % 8 == 0, 1 <= n <= 8.
 *   A [n][n] / b [n] per layer (tok_stride 0) or per token (floats per token).
 *   y_out: if not NULL, y is also stored there ([T][d] bf16), else never.
 *   Hout may equal H exactly (in place); no other overlap. X, Wo, H, Hout and
 *   y_out 16-byte aligned. Asynchronous; T == 0 is a no-op.
 */
HC_API hc_status hc_linear_then_write(const void *X, const void *Wo, const void *H, void *Hout,
                                      void *y_out, hc_dtype dt, int64_t T, int n, int64_t d,
                                      int64_t k, const float *A, int64_t A_tok_stride,
                                      const float *b, int64_t b_tok_stride, hc_stream stream);

/*
 * The write mix fused with the tensor-parallel all-reduce of the block output,
 * then the next layer's read (Hy4-preview model techniques map,
 * models.inteligile.com, the "inference kernel" row: Hy4's kernels are fused
 * and the model is served split over eight GPUs; glossary entry
 * "Hyper-connections (mHC)": streams mixed after each block). Under tensor
 * parallelism each of R ranks ends the block with a partial output y_r and
 * holds a replica of H; every rank makes this call and reads all R partials:
 *   y        = rnd( ((y_0 + y_1) + y_2) + ... + y_{R-1} )   fp32 adds in rank
 *              order, one rounding to dt (the same on every rank, so the
 *              replicas of H' and x_next stay bit-identical);
 *   then exactly hc_write_then_read(H, y, ...) with that y.
 *   y_parts: host array of R device pointers (1 <= R <= 8), the partials
 *     [T][d] of dtype dt in rank order. Each may be this device's memory or a
 *     peer's memory mapped into this process (hc_ipc_open, or an allocation
 *     on a peer-accessible device); the kernel reads them with plain loads.
 *     16-byte aligned; the library only reads them.
 *   y_out: if not NULL, y is also stored there ([T][d], dt), else never.
 *   Other arguments, layouts and checks as hc_write_then_read; no output may
 *   overlap a partial. Asynchronous on `stream`; T == 0 is a no-op.
 * The kernel never waits on another rank. The caller orders every rank's
 * writes of its partial before this call's work starts on `stream`, and any
 * later overwrite of a partial after every rank's call has finished reading
 * it (the Python layer uses a barrier on each side).
 */
HC_API hc_status hc_reduce_write_then_read(
    const void *const *y_parts, int R, const void *H, void *Hout, void *x_next, void *y_out,
    hc_dtype dt, int64_t T, int n, int64_t d, hc_mix_mode mm, const float *A, int64_t A_tok_stride,
    int K, const float *b, int64_t b_tok_stride, hc_read_mode rm, const float *a_next,
    int64_t a_tok_stride, const float *g_next, float eps, hc_stream stream);

/*
 * The reduce-scatter form of hc_reduce_write_then_read, for streams sharded
 * by token over the R ranks of a tensor-parallel group (same pages; same
 * arithmetic per token). Rank `rank` owns the contiguous tokens
 *   t0 = rank * (T_total / R) + min(rank, T_total % R),
 *   T  = T_total / R + (rank < T_total % R ? 1 : 0)
 * and, for each of them, sums the rows t0..t0+T-1 of the R partials in rank
 * order (fp32, one rounding), writes its shard of H', and stores x_next into
 * rows t0..t0+T-1 of EVERY rank's x buffer (the all-gather of x). Each rank
 * thus moves about as many bytes over NVLink as a ring all-reduce of y, and
 * does 1/R of the HBM work of the one-shot form.
 *   y_parts: R device pointers, the ranks' full partials [T_total][d].
 *   x_all:   R device pointers, the ranks' full x_next buffers [T_total][d]
 *            (x_all[rank] this rank's own); peers' may be hc_ipc_open
 *            mappings. Written only in this rank's rows.
 *   H, Hout: this rank's shard [T][n][d]; y_out: [T][d] or NULL. A, b,
 *            a_next per token index the shard's tokens (pass pointers to the
 *            shard's rows), or stride 0 for one set.
 *   1 <= R <= 8, 0 <= rank < R. Other arguments and checks as
 *   hc_reduce_write_then_read; no x_all buffer may overlap another, a
 *   partial, or this rank's inputs and outputs. T == 0 is a no-op.
 * The kernel never waits on another rank: the caller orders every partial's
 * writes before the call, and every read of x_next (or overwrite of a
 * partial) after every rank's call has finished.
 */
HC_API hc_status hc_reduce_scatter_write_then_read(
    const void *const *y_parts, int R, int rank, int64_t T_total, const void *H, void *Hout,
    void *const *x_all, void *y_out, hc_dtype dt, int n, int64_t d, hc_mix_mode mm,
    const float *A, int64_t A_tok_stride, int K, const float *b, int64_t b_tok_stride,
    hc_read_mode rm, const float *a_next, int64_t a_tok_stride, const float *g_next, float eps,
    hc_stream stream);

/*
 * Peer mappings for the partials and x buffers of the reduce calls (CUDA IPC;
 * one process per GPU). The pages have no counterpart to these; they are
 * plumbing of this library.
 *   hc_ipc_export: for a device pointer of this process, the 64-byte handle
 *     (HC_IPC_HANDLE_BYTES) of the allocation that holds it and the pointer's
 *     byte offset from that allocation's start (caching allocators hand out
 *     pointers inside larger allocations).
 *   hc_ipc_open: maps another process's allocation into this one (peer
 *     access enabled lazily) and returns its base; add the exporter's offset.
 *     A process cannot open its own handles (HC_ERR_CUDA).
 *   hc_ipc_close: unmaps a base returned by hc_ipc_open.
 * HC_ERR_INVALID_ARG on NULL arguments, HC_ERR_CUDA when the runtime refuses
 * (its message in hc_last_error). Synchronous host calls.
 */
#define HC_IPC_HANDLE_BYTES 64
HC_API hc_status hc_ipc_export(const void *dev_ptr, void *handle, uint64_t *offset);
HC_API hc_status hc_ipc_open(const void *handle, void **base);
HC_API hc_status hc_ipc_close(void *base);

/*
 * Backward pass of hc_write_then_read (training; the forward is the
 * glossary entry's mixing before and after a block with the mHC Sinkhorn
 * projection, plus the block's pre-norm). Gradients pass straight through the
 * storage rounding; every forward input is given again, unchanged.
 *   dHout [T][n][d] (gradient arriving at H', or NULL for none) and
 *   dx [T][d] (gradient arriving at x_next), dtype dt.
 *   dH [T][n][d], dy [T][d] (dtype dt) receive the gradients of H and y.
 *   dA [T][n][n], db [T][n], da [T][n] (fp32) receive per-token gradients:
 *   w.r.t. the Sinkhorn logits when mm == HC_MIX_SINKHORN_LOGITS (else the
 *   matrix) and w.r.t. the read logits when rm == HC_READ_SOFTMAX_LOGITS
 *   (else the weights). For parameters shared by all tokens (stride 0) the
 *   gradient is the sum of these over tokens.
 *   dg [d] (fp32) receives the gain gradient summed over tokens, or pass NULL;
 *   it needs g and a workspace of hc_write_then_read_backward_workspace_bytes()
 *   bytes (16-byte aligned; the sum over tokens runs in a fixed order).
 * Arithmetic: fp32 with fp64 per-token statistics and cross-warp sums. The
 * Sinkhorn backward keeps the 2K+1 iterates of a token in shared memory
 * (HC_ERR_UNSUPPORTED when K is too large for that). No output may overlap an
 * input or another output. Asynchronous; T == 0 is a no-op.
 */
HC_API hc_status hc_write_then_read_backward(
    const void *H, const void *y, hc_dtype dt, int64_t T, int n, int64_t d, hc_mix_mode mm,
    const float *A, int64_t A_tok_stride, int K, const float *b, int64_t b_tok_stride,
    hc_read_mode rm, const float *a, int64_t a_tok_stride, const float *g, float eps,
    const void *dHout, const void *dx, void *dH, void *dy, float *dA, float *db, float *da,
    float *dg, void *workspace, size_t workspace_bytes, hc_stream stream);
/* Workspace bytes the backward's gain gradient needs on the current device
 * (0 on invalid arguments). */
HC_API size_t hc_write_then_read_backward_workspace_bytes(hc_dtype dt, int64_t T, int n, int64_t d);

/*
 * hc_write_then_read_backward without a workspace argument: the pages have no
 * counterpart to this; it is an interface addition of this library for
 * callers that cannot allocate device memory when they call it -- runtimes
 * that reserve a GPU's memory up front in their own pool and have no buffer
 * to lend, and latency-critical loops where cudaMalloc, which can synchronise
 * the device, is not acceptable. The gain gradient's per-CTA partials go to a
 * 16 MiB scratch array that lives in the library's device image (one per
 * device, held until the process exits); the call allocates nothing.
 * Arguments and results are those of hc_write_then_read_backward.
 *   - The partials take hc_write_then_read_backward_workspace_bytes(dt, T, n,
 *     d) bytes; a call with dg fits when that is at most 16 MiB (16777216).
 *     Larger calls return HC_ERR_UNSUPPORTED without launching anything; use
 *     the workspace form for them. Invalid arguments get the statuses of
 *     hc_write_then_read_backward.
 *   - The scratch is shared by every call on a device: two calls whose
 *     executions overlap (different streams without ordering between them)
 *     race on it and corrupt dg. Order such calls, or use the workspace form.
 *   - The first call on a device (with dg) looks the scratch address up on
 *     the host (cudaGetSymbolAddress, with that device current) and sets
 *     kernel attributes; make that first call before any stream capture.
 *   - No part of the scratch has to start at zero.
 */
HC_API hc_status hc_write_then_read_backward_noalloc(
    const void *H, const void *y, hc_dtype dt, int64_t T, int n, int64_t d, hc_mix_mode mm,
    const float *A, int64_t A_tok_stride, int K, const float *b, int64_t b_tok_stride,
    hc_read_mode rm, const float *a, int64_t a_tok_stride, const float *g, float eps,
    const void *dHout, const void *dx, void *dH, void *dy, float *dA, float *db, float *da,
    float *dg, hc_stream stream);

/*
 * Ends of a stack ("Tencent open-sources Hy4 Preview at 770B -- Identity
 * Hyper-Connections", learnaivisually: TL;DR and the residual-design table --
 * the n streams start as copies of one; the pages do not say how they are
 * combined at the top, read here as a learned weighted sum of the streams).
 *
 * hc_expand: H[t][i][:] = x[t][:] for every stream i (a bit copy).
 *   x [T][d] in, H [T][n][d] out, dtype dt, both 16-byte aligned, no overlap.
 *
 * hc_expand_then_read: hc_expand fused with layer 0's read + pre-norm
 *   RMSNorm of the copies (arguments as hc_read_rmsnorm), so H is not read
 *   back: x_read = RMSNorm(sum_i a_i x) * g, the mix an fp32 fused
 *   multiply-add chain in stream order. x_read may equal x exactly (in place);
 *   H must not overlap x or x_read.
 *
 * hc_collapse: out[t][:] = sum_i w_i H[t][i][:], an fp32 fused multiply-add
 *   chain in stream order stored in dtype dt, no normalisation (a final norm
 *   before the head is hc_read_rmsnorm). rm == HC_READ_SOFTMAX_LOGITS turns w
 *   into weights with a softmax over the n streams first. w_tok_stride: 0 =
 *   one set for all tokens, else floats per token. out must not overlap H.
 *
 * Same shape limits and error statuses as the step calls; T == 0 is a no-op.
 */
HC_API hc_status hc_expand(const void *x, void *H, hc_dtype dt, int64_t T, int n, int64_t d,
                           hc_stream stream);
HC_API hc_status hc_expand_then_read(const void *x, void *H, void *x_read, hc_dtype dt, int64_t T,
                                     int n, int64_t d, hc_read_mode rm, const float *a,
                                     int64_t a_tok_stride, const float *g, float eps,
                                     hc_stream stream);
HC_API hc_status hc_collapse(const void *H, void *out, hc_dtype dt, int64_t T, int n, int64_t d,
                             hc_read_mode rm, const float *w, int64_t w_tok_stride,
                             hc_stream stream);

/*
 * Kernel family used by the step calls (process-wide; default HC_PATH_AUTO).
 *   HC_PATH_PIPELINED: warp-specialised kernels fed by bulk copies (TMA) into
 *     shared-memory rings, where its rings fit (for calls that normalise, two
 *     fp32 rows of d per consumer group must fit next to them: d up to 9880
 *     bf16 at n = 4). Forcing it where it does not fit returns
 *     HC_ERR_UNSUPPORTED.
 *   HC_PATH_REGISTER: register-streaming kernels (no staging).
 *   HC_PATH_AUTO: per call, the family measured faster for its sizes -- the
 *     register family for hc_read_rmsnorm, for hc_write_mix at n <= 2 and
 *     for small calls (decode-sized batches), the pipelined family for larger
 *     fused steps and writes (hc_step_path reports the choice).
 * Both families compute bit-identical results.
 */
typedef enum { HC_PATH_AUTO = 0, HC_PATH_PIPELINED = 1, HC_PATH_REGISTER = 2 } hc_path;
HC_API hc_status hc_set_path(hc_path path);
HC_API hc_path hc_get_path(void);
/*
 * The kernel family a step call of these sizes would take on the current
 * device under the current hc_set_path setting; nothing is launched.
 *   op: 0 = hc_read_rmsnorm, 1 = hc_write_mix, 2 = hc_write_then_read.
 *   *path receives HC_PATH_PIPELINED or HC_PATH_REGISTER.
 * dt, n and d are validated as by those calls; T >= 1. HC_ERR_INVALID_ARG for
 * a bad op, T < 1 or a NULL path.
 */
HC_API hc_status hc_step_path(hc_dtype dt, int op, int64_t T, int n, int64_t d, hc_path *path);

/*
 * Device-side failure report. The pipelined kernels bound every wait on
 * their shared-memory barriers (2 s of GPU time); a wait that runs out makes
 * the kernel stop, drain its copies in flight and OR a code into the current
 * device's fault word instead of hanging. This call SYNCHRONISES `stream`,
 * reads and clears that word into *code, and returns HC_ERR_DEVICE if it was
 * non-zero (HC_OK otherwise). Codes: 1 tile wait, 2 free-stage wait,
 * 4 parameter wait, 8 reduction wait, 16 drain at exit, 32 self-test.
 */
HC_API hc_status hc_device_fault(int *code, hc_stream stream);

/*
 * Self-test of the bounded waits (the mechanism, not the method; the pages
 * have no counterpart). Launches one tiny kernel whose single wait is on a
 * barrier that nothing arrives at, limited to limit_us microseconds
 * (1..100000). The wait gives up, code 32 is ORed into the device fault word
 * and the kernel returns normally: no trap, no copy in flight, the context
 * stays usable. Read the result with hc_device_fault(). Asynchronous.
 */
HC_API hc_status hc_selftest_bounded_wait(int limit_us, hc_stream stream);

/*
 * Input-dependent mixing logits (the "learned matrices" of the glossary entry
 * computed from the streams themselves; reading: an RMS-normalised linear map
 * of the token's flattened streams). For every token t:
 *   u_t = H[t] flattened to n*d values,  r_t = 1 / sqrt(mean(u_t^2) + eps),
 *   logits[t][j] = r_t * sum_k u_t[k] * W[j][k]      (j < P)
 *   H [T][n][d] bf16, W [P][n*d] bf16 (row j = the weights of logit j),
 *   logits [T][P] fp32 out. P <= 256; with P = n*n + 2n the three blocks
 *   [n*n | n | n] can feed hc_write_then_read directly as per-token Sinkhorn
 *   logits, read logits and write gains (token stride P).
 * Runs on the 5th-generation tensor cores (bf16 x bf16 -> fp32, TMEM
 * accumulator) with the sum of squares in fp64; the sum over k is in the
 * tensor core's order, so results match an exact evaluation within fp32
 * accumulation error, not bit for bit. H, W 16-byte aligned; logits 4-byte
 * aligned and disjoint from H and W. bf16 only (HC_ERR_UNSUPPORTED otherwise).
 */
HC_API hc_status hc_mix_logits(const void *H, const void *W, float *logits, hc_dtype dt,
                               int64_t T, int n, int64_t d, int P, float eps, hc_stream stream);

/* Static English text for a status code. */
HC_API const char *hc_status_string(hc_status st);

/* Details of the calling thread's most recent failed call ("" if none). The
 * pointer stays valid until the thread's next call into the library. */
HC_API const char *hc_last_error(void);

/* Library version: major * 10000 + minor * 100 + patch. */
HC_API int hc_version(void);

#ifdef __cplusplus
}
#endif

#endif /* HC_API_H */
