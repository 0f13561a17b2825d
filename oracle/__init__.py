"""CPU oracle for the Hyper-Connections residual step (ctypes over plain C).

TEST INFRASTRUCTURE: only tests/, the package smoke check and bench.py's CPU
baseline / reference arm may import this module. The product path never does,
and this module imports nothing from the product package.

Arrays are numpy. Storage dtype "bf16" arrays are np.uint16 bit patterns;
"f32" arrays are np.float32. Parameters are float32. Definitions and the
readings of the pages are documented in hc_oracle.c.
"""
from __future__ import annotations

import ctypes as C
import numpy as np

from . import build as _build

F32, BF16 = 0, 1
_DT = {"f32": F32, "bf16": BF16}
_NP = {"f32": np.float32, "bf16": np.uint16}

_lib = None


def lib():
    global _lib
    if _lib is None:
        path = _build.build()
        L = C.CDLL(path)
        i64, i32, vp, fp = C.c_int64, C.c_int, C.c_void_p, C.c_float
        sig = {
            "hco_max_threads": ([], i32),
            "hco_set_threads": ([i32], None),
            "hco_round_to": ([vp, vp, i32, i64], i32),
            "hco_sinkhorn_f32": ([vp, vp, i64, i32, i32], i32),
            "hco_sinkhorn_f64": ([vp, vp, i64, i32, i32], i32),
            "hco_softmax_f32": ([vp, vp, i64, i32], i32),
            "hco_write_mix": ([vp, vp, vp, i32, i64, i32, i64, vp, i64, vp, i64], i32),
            "hco_read_rmsnorm": ([vp, vp, i32, i64, i32, i64, vp, i64, vp, fp], i32),
            "hco_write_then_read": ([vp, vp, vp, vp, i32, i64, i32, i64, i32, vp, i64, i32,
                                     vp, i64, i32, vp, i64, vp, fp], i32),
            "hco_block_tanh": ([vp, vp, i32, i64], i32),
            "hco_mix_logits": ([vp, vp, vp, i32, i64, i32, i64, i32, fp], i32),
            "hco_single_stream_layer": ([vp, vp, i32, i64, i64, vp, fp], i32),
            "hco_expand": ([vp, vp, i32, i64, i32, i64], i32),
            "hco_linear": ([vp, vp, vp, i32, i64, i64, i64], i32),
            "hco_sinkhorn_backward": ([vp, vp, vp, i64, i32, i32], i32),
            "hco_write_then_read_backward": ([vp, vp, i32, i64, i32, i64, i32, vp, i64, i32, vp, i64,
                                              i32, vp, i64, vp, fp, vp, vp, vp, vp, vp, vp, vp, vp],
                                             i32),
            "hco_collapse": ([vp, vp, i32, i64, i32, i64, i32, vp, i64], i32),
        }
        for name, (args, res) in sig.items():
            fn = getattr(L, name)
            fn.argtypes = args
            fn.restype = res
        _lib = L
    return _lib


def _p(a):
    return None if a is None else a.ctypes.data_as(C.c_void_p)


def _chk(rc, name):
    if rc != 0:
        raise ValueError(f"oracle {name} rejected its arguments (code {rc})")


def _arr(a, dtype):
    a = np.ascontiguousarray(a, dtype=dtype)
    return a


def max_threads() -> int:
    return lib().hco_max_threads()


def set_threads(n: int) -> None:
    lib().hco_set_threads(int(n))


def round_to(x, dt: str):
    """Store fp32 values into storage dtype dt (bf16: round to nearest even)."""
    x = _arr(x, np.float32)
    out = np.empty(x.shape, dtype=_NP[dt])
    _chk(lib().hco_round_to(_p(x), _p(out), _DT[dt], x.size), "round_to")
    return out


def to_f32(x, dt: str):
    """Widen storage values to fp32 (exact)."""
    if dt == "f32":
        return np.asarray(x, dtype=np.float32)
    return (np.asarray(x, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32)


def sinkhorn(L, K: int, f64: bool = False):
    """exp then K (row pass, column pass) pairs, per n x n matrix. L: [..., n, n]."""
    dtype = np.float64 if f64 else np.float32
    L = _arr(L, dtype)
    n = L.shape[-1]
    assert L.shape[-2] == n
    T = L.size // (n * n)
    out = np.empty_like(L)
    fn = lib().hco_sinkhorn_f64 if f64 else lib().hco_sinkhorn_f32
    _chk(fn(_p(L), _p(out), T, n, int(K)), "sinkhorn")
    return out


def softmax(l):
    l = _arr(l, np.float32)
    n = l.shape[-1]
    out = np.empty_like(l)
    _chk(lib().hco_softmax_f32(_p(l), _p(out), l.size // n, n), "softmax")
    return out


def _tok_stride(p, T, per):
    """0 when one parameter set is shared by all tokens, else `per`."""
    return 0 if p.size == per else per


def write_mix(H, y, A, b, dt: str, out=None):
    """H'[t,j,:] = sum_i A[t,i,j] H[t,i,:] + b[t,j] y[t,:]. A: [n,n] or [T,n,n]."""
    H = _arr(H, _NP[dt]); y = _arr(y, _NP[dt])
    T, n, d = H.shape
    A = _arr(A, np.float32); b = _arr(b, np.float32)
    Hout = np.empty_like(H) if out is None else out
    _chk(lib().hco_write_mix(_p(H), _p(y), _p(Hout), _DT[dt], T, n, d,
                             _p(A), _tok_stride(A, T, n * n), _p(b), _tok_stride(b, T, n)),
         "write_mix")
    return Hout


def read_rmsnorm(H, a, g, eps: float, dt: str):
    """x[t,:] = RMSNorm(sum_i a[t,i] H[t,i,:]) * g. a: [n] or [T,n]; g: [d] or None."""
    H = _arr(H, _NP[dt])
    T, n, d = H.shape
    a = _arr(a, np.float32)
    g = None if g is None else _arr(g, np.float32)
    x = np.empty((T, d), dtype=_NP[dt])
    _chk(lib().hco_read_rmsnorm(_p(H), _p(x), _DT[dt], T, n, d, _p(a),
                                _tok_stride(a, T, n), _p(g), float(eps)), "read_rmsnorm")
    return x


def write_then_read(H, y, A, b, a, g, eps: float, dt: str, K: int = 0,
                    mix_logits: bool = False, read_logits: bool = False):
    """One fused HC step: write (layer l) then read + RMSNorm (layer l+1).

    Returns (H', x_next). With mix_logits, A holds Sinkhorn logits; with
    read_logits, a holds softmax logits.
    """
    H = _arr(H, _NP[dt]); y = _arr(y, _NP[dt])
    T, n, d = H.shape
    A = _arr(A, np.float32); b = _arr(b, np.float32); a = _arr(a, np.float32)
    g = None if g is None else _arr(g, np.float32)
    Hout = np.empty_like(H)
    x = np.empty((T, d), dtype=_NP[dt])
    _chk(lib().hco_write_then_read(_p(H), _p(y), _p(Hout), _p(x), _DT[dt], T, n, d,
                                   int(mix_logits), _p(A), _tok_stride(A, T, n * n), int(K),
                                   _p(b), _tok_stride(b, T, n), int(read_logits), _p(a),
                                   _tok_stride(a, T, n), _p(g), float(eps)),
         "write_then_read")
    return Hout, x


def reduce_partials(parts, dt: str):
    """The block output as the tensor-parallel all-reduce of R partials
    defines it for the fused write (a reading: the pages say the model is
    served split over eight GPUs and name no summation order): the partials,
    widened to fp32, are added left to right in rank order with an fp32
    rounding after every add (numpy float32 addition is IEEE round to nearest
    even), and the sum is rounded once to the storage dtype."""
    acc = np.array(to_f32(parts[0], dt), dtype=np.float32, copy=True)
    for p in parts[1:]:
        acc = np.add(acc, to_f32(p, dt), dtype=np.float32)
    return round_to(acc, dt)


def reduce_write_then_read(parts, H, A, b, a, g, eps: float, dt: str, K: int = 0,
                           mix_logits: bool = False, read_logits: bool = False):
    """The fused step on the all-reduced block output: (H', x_next, y) with
    y = reduce_partials(parts) and (H', x_next) = write_then_read(H, y, ...)."""
    y = reduce_partials(parts, dt)
    Hp, x = write_then_read(H, y, A, b, a, g, eps, dt, K=K, mix_logits=mix_logits,
                            read_logits=read_logits)
    return Hp, x, y


def mix_logits(H, W, eps: float, dt: str):
    """fp64 logits z[t, j] = r_t * sum_k u_t[k] W[j, k], u_t = H[t] flattened,
    r_t = 1 / sqrt(mean(u_t^2) + eps). H [T, n, d]; W [P, n*d]."""
    H = _arr(H, _NP[dt]); W = _arr(W, _NP[dt])
    T, n, d = H.shape
    P = W.shape[0]
    assert W.shape == (P, n * d)
    z = np.empty((T, P), dtype=np.float64)
    _chk(lib().hco_mix_logits(_p(H), _p(W), _p(z), _DT[dt], T, n, d, P, float(eps)), "mix_logits")
    return z


def expand(x, n: int, dt: str):
    """Stack entry: H[t, i, :] = x[t, :] for i < n. x [T, d] -> H [T, n, d]."""
    x = _arr(x, _NP[dt])
    T, d = x.shape
    H = np.empty((T, n, d), dtype=_NP[dt])
    _chk(lib().hco_expand(_p(x), _p(H), _DT[dt], T, int(n), d), "expand")
    return H


def expand_then_read(x, n: int, a, g, eps: float, dt: str, read_logits: bool = False):
    """Stack entry followed by layer 0's read: (expand(x), RMSNorm(sum_i a_i H_i) g)
    of the expanded streams; with read_logits, a holds softmax logits."""
    H = expand(x, n, dt)
    w = softmax(a) if read_logits else a
    return H, read_rmsnorm(H, w, g, eps, dt)


def collapse(H, w, dt: str, read_logits: bool = False):
    """Stack exit: out[t] = sum_i w_i H[t, i] (fmaf chain, stored in dt).
    w: [n] or [T, n]; with read_logits, w holds softmax logits."""
    H = _arr(H, _NP[dt])
    T, n, d = H.shape
    w = _arr(w, np.float32)
    out = np.empty((T, d), dtype=_NP[dt])
    _chk(lib().hco_collapse(_p(H), _p(out), _DT[dt], T, n, d, int(read_logits), _p(w),
                            _tok_stride(w, T, n)), "collapse")
    return out


def linear(X, W, dt: str):
    """fp64 y[t, c] = sum_k X[t, k] W[c, k]. X [T, k], W [d, k] storage arrays."""
    X = _arr(X, _NP[dt]); W = _arr(W, _NP[dt])
    T, k = X.shape
    d = W.shape[0]
    assert W.shape == (d, k)
    y = np.empty((T, d), dtype=np.float64)
    _chk(lib().hco_linear(_p(X), _p(W), _p(y), _DT[dt], T, k, d), "linear")
    return y


def sinkhorn_backward(L, dA, K: int):
    """fp64 gradient w.r.t. the logits L [..., n, n] of the Sinkhorn projection
    (exp, then K row/column pairs), given the gradient dA w.r.t. its output."""
    L = _arr(L, np.float32)
    dA = _arr(dA, np.float64)
    n = L.shape[-1]
    T = L.size // (n * n)
    dL = np.empty(L.shape, dtype=np.float64)
    _chk(lib().hco_sinkhorn_backward(_p(L), _p(dA), _p(dL), T, n, int(K)), "sinkhorn_backward")
    return dL


def write_then_read_backward(H, y, A, b, a, g, eps: float, dt: str, dHout, dx, K: int = 0,
                             mix_logits: bool = False, read_logits: bool = False, want_dg=True):
    """fp64 gradients of the fused step (straight through the storage rounding).
    dHout [T, n, d] (or None) and dx [T, d] are the upstream gradients. Returns
    dict(dH, dy, dA, db, da, dg): dA / db / da per token ([T, n, n], [T, n],
    [T, n]; with mix_logits / read_logits, w.r.t. the logits); dg [d] summed
    over tokens (None if g is None or not want_dg)."""
    H = _arr(H, _NP[dt]); y = _arr(y, _NP[dt])
    T, n, d = H.shape
    A = _arr(A, np.float32); b = _arr(b, np.float32); a = _arr(a, np.float32)
    g = None if g is None else _arr(g, np.float32)
    dHout = None if dHout is None else _arr(dHout, np.float64)
    dx = _arr(dx, np.float64)
    out = dict(dH=np.empty((T, n, d)), dy=np.empty((T, d)), dA=np.empty((T, n, n)),
               db=np.empty((T, n)), da=np.empty((T, n)),
               dg=np.empty(d) if (g is not None and want_dg) else None)
    _chk(lib().hco_write_then_read_backward(
        _p(H), _p(y), _DT[dt], T, n, d, int(mix_logits), _p(A), _tok_stride(A, T, n * n), int(K),
        _p(b), _tok_stride(b, T, n), int(read_logits), _p(a), _tok_stride(a, T, n), _p(g),
        float(eps), _p(dHout), _p(dx), _p(out["dH"]), _p(out["dy"]), _p(out["dA"]), _p(out["db"]),
        _p(out["da"]), _p(out["dg"])), "write_then_read_backward")
    return out


def block_tanh(x, dt: str):
    """Harness stand-in for the block body: y = round(tanh(x))."""
    x = _arr(x, _NP[dt])
    y = np.empty_like(x)
    _chk(lib().hco_block_tanh(_p(x), _p(y), _DT[dt], x.size), "block_tanh")
    return y


def single_stream_layer(x, g, eps: float, dt: str):
    """x + tanh(RMSNorm(x) * g): the one-stream pre-norm residual layer."""
    x = _arr(x, _NP[dt])
    T, d = x.shape
    g = None if g is None else _arr(g, np.float32)
    out = np.empty_like(x)
    _chk(lib().hco_single_stream_layer(_p(x), _p(out), _DT[dt], T, d, _p(g), float(eps)),
         "single_stream_layer")
    return out
