"""ctypes binding of libhc_b200.so (include/hc_api.h).

Argument marshalling only: tensors are checked for device, dtype, shape and
contiguity, turned into raw pointers plus token strides, and the call is
enqueued on torch's current CUDA stream. Every step of the HC computation runs
in the library's kernels; there is no fallback. If the library is missing or
fails to load, every call raises.
"""
from __future__ import annotations

import ctypes as C
import os

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libhc_b200.so")

HC_OK, HC_ERR_INVALID_ARG, HC_ERR_UNSUPPORTED, HC_ERR_MISALIGNED = 0, 1, 2, 3
HC_ERR_ALIAS, HC_ERR_CUDA, HC_ERR_DEVICE = 4, 5, 6
HC_F32, HC_BF16 = 0, 1
PATH_AUTO, PATH_PIPELINED, PATH_REGISTER = 0, 1, 2
MIX_MATRIX, MIX_SINKHORN_LOGITS = 0, 1
READ_WEIGHTS, READ_SOFTMAX_LOGITS = 0, 1

_DT = {torch.float32: HC_F32, torch.bfloat16: HC_BF16}

# C signatures of the entry points in include/hc_api.h
_i64, _i32, _vp, _f32 = C.c_int64, C.c_int, C.c_void_p, C.c_float
SIGNATURES = {
    "hc_sinkhorn": ([_vp, _vp, _i64, _i32, _i32, _vp], _i32),
    "hc_read_rmsnorm": ([_vp, _vp, _i32, _i64, _i32, _i64, _i32, _vp, _i64, _vp, _f32, _vp], _i32),
    "hc_write_mix": ([_vp, _vp, _vp, _i32, _i64, _i32, _i64, _i32, _vp, _i64, _i32, _vp, _i64,
                      _vp], _i32),
    "hc_write_then_read": ([_vp, _vp, _vp, _vp, _i32, _i64, _i32, _i64, _i32, _vp, _i64, _i32,
                            _vp, _i64, _i32, _vp, _i64, _vp, _f32, _vp], _i32),
    "hc_set_path": ([_i32], _i32),
    "hc_get_path": ([], _i32),
    "hc_step_path": ([_i32, _i32, _i64, _i32, _i64, C.POINTER(_i32)], _i32),
    "hc_device_fault": ([C.POINTER(_i32), _vp], _i32),
    "hc_selftest_bounded_wait": ([_i32, _vp], _i32),
    "hc_mix_logits": ([_vp, _vp, _vp, _i32, _i64, _i32, _i64, _i32, _f32, _vp], _i32),
    "hc_expand": ([_vp, _vp, _i32, _i64, _i32, _i64, _vp], _i32),
    "hc_write_then_read_backward": ([_vp, _vp, _i32, _i64, _i32, _i64, _i32, _vp, _i64, _i32, _vp,
                                     _i64, _i32, _vp, _i64, _vp, _f32, _vp, _vp, _vp, _vp, _vp,
                                     _vp, _vp, _vp, _vp, C.c_size_t, _vp], _i32),
    "hc_write_then_read_backward_workspace_bytes": ([_i32, _i64, _i32, _i64], C.c_size_t),
    "hc_write_then_read_backward_noalloc": ([_vp, _vp, _i32, _i64, _i32, _i64, _i32, _vp, _i64, _i32,
                                             _vp, _i64, _i32, _vp, _i64, _vp, _f32, _vp, _vp, _vp,
                                             _vp, _vp, _vp, _vp, _vp, _vp], _i32),
    "hc_linear_then_write": ([_vp, _vp, _vp, _vp, _vp, _i32, _i64, _i32, _i64, _i64, _vp, _i64,
                              _vp, _i64, _vp], _i32),
    "hc_expand_then_read": ([_vp, _vp, _vp, _i32, _i64, _i32, _i64, _i32, _vp, _i64, _vp, _f32,
                             _vp], _i32),
    "hc_collapse": ([_vp, _vp, _i32, _i64, _i32, _i64, _i32, _vp, _i64, _vp], _i32),
    "hc_reduce_write_then_read": ([_vp, _i32, _vp, _vp, _vp, _vp, _i32, _i64, _i32, _i64, _i32, _vp,
                                   _i64, _i32, _vp, _i64, _i32, _vp, _i64, _vp, _f32, _vp], _i32),
    "hc_reduce_scatter_write_then_read": ([_vp, _i32, _i32, _i64, _vp, _vp, _vp, _vp, _i32, _i32,
                                           _i64, _i32, _vp, _i64, _i32, _vp, _i64, _i32, _vp, _i64,
                                           _vp, _f32, _vp], _i32),
    "hc_ipc_export": ([_vp, _vp, C.POINTER(C.c_uint64)], _i32),
    "hc_ipc_open": ([_vp, C.POINTER(_vp)], _i32),
    "hc_ipc_close": ([_vp], _i32),
    "hc_status_string": ([_i32], C.c_char_p),
    "hc_last_error": ([], C.c_char_p),
    "hc_version": ([], _i32),
}


class HCError(RuntimeError):
    def __init__(self, status: int, detail: str):
        super().__init__(f"{status_string(status)} ({status}): {detail}")
        self.status = status


_lib = None


def lib():
    """Load libhc_b200.so (raises if it is missing: build it first with
    `python -m hyper_connections_stream_b200.build`)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise ImportError(f"libhc_b200.so not found at {LIB_PATH}; build it with "
                              "`python -m hyper_connections_stream_b200.build`")
        L = C.CDLL(LIB_PATH)
        for name, (args, res) in SIGNATURES.items():
            fn = getattr(L, name)
            fn.argtypes = args
            fn.restype = res
        _lib = L
    return _lib


def status_string(st: int) -> str:
    return lib().hc_status_string(int(st)).decode()


def _check(st: int):
    if st != HC_OK:
        raise HCError(st, lib().hc_last_error().decode())


def _ptr(t):
    return None if t is None else C.c_void_p(t.data_ptr())


def _stream(device):
    return C.c_void_p(torch.cuda.current_stream(device).cuda_stream)


def _need_cuda(name, t, dtype=None):
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if dtype is not None and t.dtype != dtype:
        raise ValueError(f"{name} must be {dtype}, got {t.dtype}")


def _need_out(name, t, shape, dtype):
    """An output tensor: CUDA, contiguous, of exactly this shape and dtype (the
    library writes shape-many elements through the raw pointer)."""
    _need_cuda(name, t, dtype)
    if tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} must be {tuple(shape)}, got {tuple(t.shape)}")


def _need_gain(name, g, d):
    if g is not None:
        _need_cuda(name, g, torch.float32)
        if tuple(g.shape) != (d,):
            raise ValueError(f"{name} must be [d]")


def _tok_layout(name, p, T, per_shape):
    """Token stride in floats of a shared ([*per_shape], contiguous) or
    per-token ([T, *per_shape]) parameter: 0 when shared. A per-token
    parameter may be a view whose tokens are `stride(0)` floats apart as long
    as each token's set is contiguous (e.g. a slice of the [T, P] output of
    mix_logits); with T == 0 nothing of it is read."""
    per = 1
    for s in per_shape:
        per *= s
    if tuple(p.shape) == tuple(per_shape):
        if not p.is_contiguous():
            raise ValueError(f"{name} must be contiguous")
        return 0
    if tuple(p.shape) == (T, *per_shape):
        if T > 0 and not p[0].is_contiguous():
            raise ValueError(f"{name}: each token's values must be contiguous")
        return p.stride(0) if T > 1 else per
    raise ValueError(f"{name} must have shape {tuple(per_shape)} or {(T, *per_shape)}, "
                     f"got {tuple(p.shape)}")


def _tok_param(name, p, T, per_shape):
    """A float32 CUDA parameter, shared or per token -> its token stride."""
    if not isinstance(p, torch.Tensor) or not p.is_cuda or p.dtype != torch.float32:
        raise ValueError(f"{name} must be a float32 CUDA tensor")
    return _tok_layout(name, p, T, per_shape)


def _streams_shape(H):
    if H.dim() != 3:
        raise ValueError(f"H must be [T, n, d], got {tuple(H.shape)}")
    if H.dtype not in _DT:
        raise ValueError(f"H must be float32 or bfloat16, got {H.dtype}")
    return H.shape


def set_path(path: int) -> None:
    """Choose the kernel family process-wide: PATH_AUTO, PATH_PIPELINED (TMA-fed
    ring) or PATH_REGISTER (register streaming). Results are identical."""
    _check(lib().hc_set_path(int(path)))


def get_path() -> int:
    return int(lib().hc_get_path())


STEP_OPS = {"read": 0, "write": 1, "fused": 2}


def step_path(op: str, T: int, n: int, d: int, dtype=torch.bfloat16) -> int:
    """The kernel family (PATH_PIPELINED or PATH_REGISTER) a read, write or
    fused step call of these sizes takes on the current device under the
    current set_path setting; nothing is launched."""
    out = C.c_int(0)
    _check(lib().hc_step_path(_DT[dtype], STEP_OPS[op], int(T), int(n), int(d), C.byref(out)))
    return int(out.value)


def device_fault(device=None) -> int:
    """Synchronise the current stream and return (and clear) the device fault
    word: 0 when no kernel gave up on a bounded wait."""
    code = C.c_int(0)
    st = lib().hc_device_fault(C.byref(code), _stream(device))
    if st not in (HC_OK, HC_ERR_DEVICE):
        _check(st)
    return int(code.value)


def mix_logits(H, W, *, eps: float = 1e-6, out=None):
    """Per-token mixing logits on the tensor cores: out[t, j] = r_t * (u_t . W[j])
    with u_t = H[t] flattened and r_t its inverse RMS. H [T, n, d] bf16,
    W [P, n*d] bf16 -> out [T, P] fp32."""
    _need_cuda("H", H, torch.bfloat16)
    T, n, d = _streams_shape(H)
    _need_cuda("W", W, torch.bfloat16)
    if W.dim() != 2 or W.shape[1] != n * d:
        raise ValueError(f"W must be [P, n*d = {n * d}], got {tuple(W.shape)}")
    P = W.shape[0]
    out = torch.empty((T, P), dtype=torch.float32, device=H.device) if out is None else out
    _need_out("out", out, (T, P), torch.float32)
    _check(lib().hc_mix_logits(_ptr(H), _ptr(W), _ptr(out), HC_BF16, T, n, d, P, float(eps),
                               _stream(H.device)))
    return out


def selftest_bounded_wait(limit_us: int = 1000, device=None) -> None:
    """Launch the bounded-wait self-test (see hc_selftest_bounded_wait)."""
    _check(lib().hc_selftest_bounded_wait(int(limit_us), _stream(device)))


def sinkhorn(logits: torch.Tensor, K: int, out: torch.Tensor | None = None) -> torch.Tensor:
    """Doubly stochastic projection of [..., n, n] fp32 logits: exp, then K
    (row, column) normalisation pairs."""
    _need_cuda("logits", logits, torch.float32)
    n = logits.shape[-1]
    if logits.dim() < 2 or logits.shape[-2] != n:
        raise ValueError("logits must be [..., n, n]")
    T = logits.numel() // (n * n) if n else 0
    out = torch.empty_like(logits) if out is None else out
    _need_out("out", out, tuple(logits.shape), torch.float32)
    _check(lib().hc_sinkhorn(_ptr(logits), _ptr(out), T, n, int(K), _stream(logits.device)))
    return out


def read_rmsnorm(H, a, g=None, *, eps: float = 1e-6, read: int = READ_WEIGHTS, x=None):
    """x = RMSNorm(sum_i a_i H_i) * g. H [T,n,d]; a [n] or [T,n] (weights or,
    with read=READ_SOFTMAX_LOGITS, logits); g [d] fp32 or None."""
    _need_cuda("H", H)
    T, n, d = _streams_shape(H)
    a_s = _tok_param("a", a, T, (n,))
    if g is not None:
        _need_cuda("g", g, torch.float32)
        if tuple(g.shape) != (d,):
            raise ValueError("g must be [d]")
    x = torch.empty((T, d), dtype=H.dtype, device=H.device) if x is None else x
    _need_out("x", x, (T, d), H.dtype)
    _check(lib().hc_read_rmsnorm(_ptr(H), _ptr(x), _DT[H.dtype], T, n, d, int(read), _ptr(a),
                                 a_s, _ptr(g), float(eps), _stream(H.device)))
    return x


def write_mix(H, y, A, b, *, mix: int = MIX_MATRIX, K: int = 0, out=None):
    """H'_j = sum_i A[i,j] H_i + b_j y. A [n,n] or [T,n,n] (matrix or, with
    mix=MIX_SINKHORN_LOGITS, logits projected by K Sinkhorn pairs); b [n] or
    [T,n]. out may be H (in place)."""
    _need_cuda("H", H)
    T, n, d = _streams_shape(H)
    _need_cuda("y", y, H.dtype)
    if tuple(y.shape) != (T, d):
        raise ValueError("y must be [T, d]")
    A_s = _tok_param("A", A, T, (n, n))
    b_s = _tok_param("b", b, T, (n,))
    out = torch.empty_like(H) if out is None else out
    _need_out("out", out, (T, n, d), H.dtype)
    _check(lib().hc_write_mix(_ptr(H), _ptr(y), _ptr(out), _DT[H.dtype], T, n, d, int(mix),
                              _ptr(A), A_s, int(K), _ptr(b), b_s, _stream(H.device)))
    return out


def write_then_read(H, y, A, b, a_next, g_next=None, *, eps: float = 1e-6,
                    mix: int = MIX_MATRIX, K: int = 0, read: int = READ_WEIGHTS,
                    out=None, x_next=None):
    """Fused: layer l's write, then layer l+1's read + RMSNorm of the stored H'.
    Returns (H', x_next)."""
    _need_cuda("H", H)
    T, n, d = _streams_shape(H)
    _need_cuda("y", y, H.dtype)
    if tuple(y.shape) != (T, d):
        raise ValueError("y must be [T, d]")
    A_s = _tok_param("A", A, T, (n, n))
    b_s = _tok_param("b", b, T, (n,))
    a_s = _tok_param("a_next", a_next, T, (n,))
    if g_next is not None:
        _need_cuda("g_next", g_next, torch.float32)
        if tuple(g_next.shape) != (d,):
            raise ValueError("g_next must be [d]")
    out = torch.empty_like(H) if out is None else out
    x_next = torch.empty((T, d), dtype=H.dtype, device=H.device) if x_next is None else x_next
    _need_out("out", out, (T, n, d), H.dtype)
    _need_out("x_next", x_next, (T, d), H.dtype)
    _check(lib().hc_write_then_read(_ptr(H), _ptr(y), _ptr(out), _ptr(x_next), _DT[H.dtype],
                                    T, n, d, int(mix), _ptr(A), A_s, int(K), _ptr(b), b_s,
                                    int(read), _ptr(a_next), a_s, _ptr(g_next), float(eps),
                                    _stream(H.device)))
    return out, x_next


def reduce_write_then_read(parts, H, A, b, a_next, g_next=None, *, eps: float = 1e-6,
                           mix: int = MIX_MATRIX, K: int = 0, read: int = READ_WEIGHTS,
                           out=None, x_next=None, y_out=None):
    """The fused step on the tensor-parallel all-reduce of the block output:
    y = rnd(sum of the R partials in rank order, fp32), then
    (H', x_next) = write_then_read(H, y, ...). `parts` lists the R partials in
    rank order, each a [T, d] CUDA tensor of H's dtype or an int device
    address (a peer mapping from dist.PeerPartials). y is stored only into
    y_out when given. Returns (H', x_next). The call does not order the
    partials' writes or overwrites against other ranks; dist.reduce_step
    does."""
    _need_cuda("H", H)
    T, n, d = _streams_shape(H)
    R = len(parts)
    if not 1 <= R <= 8:
        raise ValueError("1 <= len(parts) <= 8")
    addrs = []
    for r, q in enumerate(parts):
        if isinstance(q, int):
            addrs.append(q)
        else:
            _need_cuda(f"parts[{r}]", q, H.dtype)
            if tuple(q.shape) != (T, d):
                raise ValueError(f"parts[{r}] must be [T, d]")
            addrs.append(q.data_ptr())
    A_s = _tok_param("A", A, T, (n, n))
    b_s = _tok_param("b", b, T, (n,))
    a_s = _tok_param("a_next", a_next, T, (n,))
    if g_next is not None:
        _need_cuda("g_next", g_next, torch.float32)
        if tuple(g_next.shape) != (d,):
            raise ValueError("g_next must be [d]")
    out = torch.empty_like(H) if out is None else out
    x_next = torch.empty((T, d), dtype=H.dtype, device=H.device) if x_next is None else x_next
    _need_out("out", out, (T, n, d), H.dtype)
    _need_out("x_next", x_next, (T, d), H.dtype)
    if y_out is not None:
        _need_out("y_out", y_out, (T, d), H.dtype)
    arr = (C.c_void_p * R)(*addrs)
    _check(lib().hc_reduce_write_then_read(C.cast(arr, C.c_void_p), R, _ptr(H), _ptr(out),
                                           _ptr(x_next), _ptr(y_out), _DT[H.dtype], T, n, d,
                                           int(mix), _ptr(A), A_s, int(K), _ptr(b), b_s,
                                           int(read), _ptr(a_next), a_s, _ptr(g_next),
                                           float(eps), _stream(H.device)))
    return out, x_next


def _addrs(name, bufs, shape, dtype):
    out = []
    for r, q in enumerate(bufs):
        if isinstance(q, int):
            out.append(q)
        else:
            _need_cuda(f"{name}[{r}]", q, dtype)
            if tuple(q.shape) != shape:
                raise ValueError(f"{name}[{r}] must be {list(shape)}")
            out.append(q.data_ptr())
    return out


def reduce_scatter_write_then_read(parts, x_all, rank: int, H, A, b, a_next, g_next=None, *,
                                   eps: float = 1e-6, mix: int = MIX_MATRIX, K: int = 0,
                                   read: int = READ_WEIGHTS, out=None, y_out=None,
                                   T_total: int | None = None):
    """The reduce-scatter form: H is this rank's token shard [T_r, n, d] of
    the group's streams; parts and x_all list the R ranks' full [T, d] partials
    and x_next buffers (tensors or int device addresses). Reduces the rank's
    rows of the partials, writes its shard of H' (returned) and stores x_next
    for its rows into every x_all buffer. T is inferred from the buffers
    passed as tensors, or given as T_total when all are addresses."""
    _need_cuda("H", H)
    Tr, n, d = _streams_shape(H)
    R = len(parts)
    if not 1 <= R <= 8 or len(x_all) != R:
        raise ValueError("1 <= len(parts) == len(x_all) <= 8")
    T = None
    for q in list(parts) + list(x_all):
        if not isinstance(q, int):
            T = q.shape[0]
            break
    if T is None:
        T = T_total
    elif T_total is not None and int(T_total) != T:
        raise ValueError(f"T_total = {T_total} but the buffers hold {T} rows")
    if T is None:
        raise ValueError("pass T_total, or at least one partial or x buffer as a tensor")
    T = int(T)
    if not 0 <= rank < R:
        raise ValueError("0 <= rank < len(parts)")
    base, extra = divmod(T, R)
    if Tr != base + (1 if rank < extra else 0):
        raise ValueError(f"H holds {Tr} tokens; rank {rank} of {R} owns {base + (rank < extra)} of {T}")
    pa = _addrs("parts", parts, (T, d), H.dtype)
    xa = _addrs("x_all", x_all, (T, d), H.dtype)
    A_s = _tok_param("A", A, Tr, (n, n))
    b_s = _tok_param("b", b, Tr, (n,))
    a_s = _tok_param("a_next", a_next, Tr, (n,))
    if g_next is not None:
        _need_cuda("g_next", g_next, torch.float32)
        if tuple(g_next.shape) != (d,):
            raise ValueError("g_next must be [d]")
    out = torch.empty_like(H) if out is None else out
    _need_out("out", out, (Tr, n, d), H.dtype)
    if y_out is not None:
        _need_out("y_out", y_out, (Tr, d), H.dtype)
    parr = (C.c_void_p * R)(*pa)
    xarr = (C.c_void_p * R)(*xa)
    _check(lib().hc_reduce_scatter_write_then_read(
        C.cast(parr, C.c_void_p), R, int(rank), T, _ptr(H), _ptr(out), C.cast(xarr, C.c_void_p),
        _ptr(y_out), _DT[H.dtype], n, d, int(mix), _ptr(A), A_s, int(K), _ptr(b), b_s, int(read),
        _ptr(a_next), a_s, _ptr(g_next), float(eps), _stream(H.device)))
    return out


def ipc_export(t: torch.Tensor):
    """(64-byte handle, byte offset) of the CUDA allocation holding t."""
    handle = C.create_string_buffer(64)
    off = C.c_uint64(0)
    _check(lib().hc_ipc_export(C.c_void_p(t.data_ptr()), handle, C.byref(off)))
    return handle.raw, int(off.value)


def ipc_open(handle: bytes) -> int:
    """Base address of another process's allocation, mapped into this one."""
    buf = C.create_string_buffer(bytes(handle), 64)
    base = C.c_void_p(0)
    _check(lib().hc_ipc_open(buf, C.byref(base)))
    return int(base.value)


def ipc_close(base: int) -> None:
    _check(lib().hc_ipc_close(C.c_void_p(base)))


def expand(x, n: int, *, out=None):
    """Stack entry: H[t, i, :] = x[t, :] for the n streams. x [T, d] -> H [T, n, d]."""
    _need_cuda("x", x)
    if x.dim() != 2 or x.dtype not in _DT:
        raise ValueError("x must be [T, d] float32 or bfloat16")
    T, d = x.shape
    out = torch.empty((T, n, d), dtype=x.dtype, device=x.device) if out is None else out
    _need_out("out", out, (T, n, d), x.dtype)
    _check(lib().hc_expand(_ptr(x), _ptr(out), _DT[x.dtype], T, int(n), d, _stream(x.device)))
    return out


def expand_then_read(x, n: int, a, g=None, *, eps: float = 1e-6, read: int = READ_WEIGHTS,
                     out=None, x_read=None):
    """Stack entry fused with layer 0's read: H = n copies of x, and
    x_read = RMSNorm(sum_i a_i x) * g. Returns (H, x_read); x_read may be x."""
    _need_cuda("x", x)
    if x.dim() != 2 or x.dtype not in _DT:
        raise ValueError("x must be [T, d] float32 or bfloat16")
    T, d = x.shape
    a_s = _tok_param("a", a, T, (int(n),))
    _need_gain("g", g, d)
    out = torch.empty((T, n, d), dtype=x.dtype, device=x.device) if out is None else out
    x_read = torch.empty_like(x) if x_read is None else x_read
    _need_out("out", out, (T, n, d), x.dtype)
    _need_out("x_read", x_read, (T, d), x.dtype)
    _check(lib().hc_expand_then_read(_ptr(x), _ptr(out), _ptr(x_read), _DT[x.dtype], T, int(n), d,
                                     int(read), _ptr(a), a_s, _ptr(g), float(eps),
                                     _stream(x.device)))
    return out, x_read


def collapse(H, w, *, read: int = READ_WEIGHTS, out=None):
    """Stack exit: out = sum_i w_i H_i (no normalisation). w [n] or [T, n]
    (weights or, with read=READ_SOFTMAX_LOGITS, logits)."""
    _need_cuda("H", H)
    T, n, d = _streams_shape(H)
    w_s = _tok_param("w", w, T, (n,))
    out = torch.empty((T, d), dtype=H.dtype, device=H.device) if out is None else out
    _need_out("out", out, (T, d), H.dtype)
    _check(lib().hc_collapse(_ptr(H), _ptr(out), _DT[H.dtype], T, n, d, int(read), _ptr(w), w_s,
                             _stream(H.device)))
    return out


def linear_then_write(X, Wo, H, A, b, *, out=None, y_out=None):
    """The block's output projection fused with the write mix:
    y = bf16(X Wo^T) on the tensor cores, H'_j = sum_i A[i,j] H_i + b_j y.
    X [T, k], Wo [d, k], H [T, n, d], all bf16; A [n, n] or [T, n, n] (a
    matrix); b [n] or [T, n]. y is stored only if y_out is given. out may be H."""
    _need_cuda("X", X, torch.bfloat16)
    _need_cuda("Wo", Wo, torch.bfloat16)
    _need_cuda("H", H, torch.bfloat16)
    T, n, d = _streams_shape(H)
    if X.dim() != 2 or X.shape[0] != T:
        raise ValueError(f"X must be [T = {T}, k], got {tuple(X.shape)}")
    k = X.shape[1]
    if tuple(Wo.shape) != (d, k):
        raise ValueError(f"Wo must be [d = {d}, k = {k}], got {tuple(Wo.shape)}")
    A_s = _tok_param("A", A, T, (n, n))
    b_s = _tok_param("b", b, T, (n,))
    out = torch.empty_like(H) if out is None else out
    _need_out("out", out, (T, n, d), torch.bfloat16)
    if y_out is not None:
        _need_out("y_out", y_out, (T, d), torch.bfloat16)
    _check(lib().hc_linear_then_write(_ptr(X), _ptr(Wo), _ptr(H), _ptr(out), _ptr(y_out), HC_BF16,
                                      T, n, d, k, _ptr(A), A_s, _ptr(b), b_s, _stream(H.device)))
    return out


def write_then_read_backward(H, y, A, b, a, g, dHout, dx, *, eps: float = 1e-6,
                             mix: int = MIX_MATRIX, K: int = 0, read: int = READ_WEIGHTS,
                             want_dg: bool = True, workspace=None):
    """Backward of write_then_read. dHout [T, n, d] (or None) and dx [T, d] are
    the gradients arriving at H' and x_next. Returns a dict with dH, dy (dtype
    of H), dA [T, n, n], db [T, n], da [T, n] (fp32, per token; w.r.t. the
    logits in the Sinkhorn / softmax modes) and dg [d] (summed over tokens, or
    None). The gain gradient's workspace is allocated here unless given."""
    _need_cuda("H", H)
    T, n, d = _streams_shape(H)
    _need_cuda("y", y, H.dtype)
    _need_cuda("dx", dx, H.dtype)
    if tuple(y.shape) != (T, d) or tuple(dx.shape) != (T, d):
        raise ValueError("y and dx must be [T, d]")
    if dHout is not None:
        _need_out("dHout", dHout, (T, n, d), H.dtype)
    A_s = _tok_param("A", A, T, (n, n))
    b_s = _tok_param("b", b, T, (n,))
    a_s = _tok_param("a", a, T, (n,))
    _need_gain("g", g, d)
    dev = H.device
    out = dict(dH=torch.empty_like(H), dy=torch.empty_like(y),
               dA=torch.empty((T, n, n), dtype=torch.float32, device=dev),
               db=torch.empty((T, n), dtype=torch.float32, device=dev),
               da=torch.empty((T, n), dtype=torch.float32, device=dev),
               dg=torch.empty((d,), dtype=torch.float32, device=dev) if (g is not None and want_dg)
               else None)
    ws_bytes = 0
    if out["dg"] is not None:
        need = int(lib().hc_write_then_read_backward_workspace_bytes(_DT[H.dtype], T, n, d)) if T else 0
        if workspace is None:
            workspace = torch.empty((max(need, 16),), dtype=torch.uint8, device=dev)
        _need_cuda("workspace", workspace, torch.uint8)
        ws_bytes = workspace.numel()
    _check(lib().hc_write_then_read_backward(
        _ptr(H), _ptr(y), _DT[H.dtype], T, n, d, int(mix), _ptr(A), A_s, int(K), _ptr(b), b_s,
        int(read), _ptr(a), a_s, _ptr(g), float(eps), _ptr(dHout), _ptr(dx), _ptr(out["dH"]),
        _ptr(out["dy"]), _ptr(out["dA"]), _ptr(out["db"]), _ptr(out["da"]), _ptr(out["dg"]),
        _ptr(workspace) if out["dg"] is not None else None, ws_bytes, _stream(dev)))
    return out


def write_then_read_backward_noalloc(H, y, A, b, a, g, dHout, dx, *, eps: float = 1e-6,
                                     mix: int = MIX_MATRIX, K: int = 0, read: int = READ_WEIGHTS,
                                     out=None):
    """write_then_read_backward through hc_write_then_read_backward_noalloc
    (the gain gradient's scratch is the library's static device array). out,
    if given, is a dict of preallocated outputs as write_then_read_backward
    returns them."""
    _need_cuda("H", H)
    T, n, d = _streams_shape(H)
    _need_cuda("y", y, H.dtype)
    _need_cuda("dx", dx, H.dtype)
    if tuple(y.shape) != (T, d) or tuple(dx.shape) != (T, d):
        raise ValueError("y and dx must be [T, d]")
    if dHout is not None:
        _need_out("dHout", dHout, (T, n, d), H.dtype)
    A_s = _tok_param("A", A, T, (n, n))
    b_s = _tok_param("b", b, T, (n,))
    a_s = _tok_param("a", a, T, (n,))
    _need_gain("g", g, d)
    dev = H.device
    if out is None:
        out = dict(dH=torch.empty_like(H), dy=torch.empty_like(y),
                   dA=torch.empty((T, n, n), dtype=torch.float32, device=dev),
                   db=torch.empty((T, n), dtype=torch.float32, device=dev),
                   da=torch.empty((T, n), dtype=torch.float32, device=dev),
                   dg=torch.empty((d,), dtype=torch.float32, device=dev) if g is not None else None)
    _need_out("dH", out["dH"], (T, n, d), H.dtype)
    _need_out("dy", out["dy"], (T, d), H.dtype)
    _need_out("dA", out["dA"], (T, n, n), torch.float32)
    _need_out("db", out["db"], (T, n), torch.float32)
    _need_out("da", out["da"], (T, n), torch.float32)
    if out["dg"] is not None:
        _need_out("dg", out["dg"], (d,), torch.float32)
    _check(lib().hc_write_then_read_backward_noalloc(
        _ptr(H), _ptr(y), _DT[H.dtype], T, n, d, int(mix), _ptr(A), A_s, int(K), _ptr(b), b_s,
        int(read), _ptr(a), a_s, _ptr(g), float(eps), _ptr(dHout), _ptr(dx), _ptr(out["dH"]),
        _ptr(out["dy"]), _ptr(out["dA"]), _ptr(out["db"]), _ptr(out["da"]), _ptr(out["dg"]),
        _stream(dev)))
    return out
