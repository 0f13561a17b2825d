"""GPU parity of the write fused with the tensor-parallel all-reduce of the
block output (hc_reduce_write_then_read) against the oracle.

R partial buffers of one GPU stand for the R ranks' buffers: the kernel reads
them with the same plain loads it issues on peer memory, and nothing in it
waits on another rank, so one GPU runs the whole computation of every rank.
The oracle sums the partials in rank order in fp32, rounds once, and runs its
fused step on that y.

Every case runs under each kernel family (chosen by size, pipelined, register
streaming). The pipelined kernel stages partials in this GPU's memory with
bulk copies and reads any other partial with plain loads; a case with some
partials in managed memory (which the library does not stage) covers the
plain-load branch on one GPU.

Bars: y bit-exact always (no parameter enters it); H' and x_next bit-exact
with the matrix and weights given (the same fp32 chains on both sides); with
Sinkhorn and softmax logits within the fused step's bars (2e-2 bf16 / 1e-5
fp32, relative with the per-token rms floor), and for bf16 storage > 99.9 % of
H' bit-identical (exp differs by ulps between libm and CUDA; fp32 storage
keeps those differences in the last bit of most elements).
"""
from __future__ import annotations

import numpy as np
import pytest
import torch

import hc_inputs as gen
import oracle
from tests._parity import TORCH_DT, assert_close, f32_dev, to_dev, to_host

pytestmark = pytest.mark.gpu
EPS = 1e-6


@pytest.fixture(scope="module", params=["auto", "pipelined", "register"])
def hc(request):
    """The binding with the kernel family chosen by call size, or forced to the
    pipelined (bulk-copy rings) or the register-streaming kernel."""
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from hyper_connections_stream_b200 import build
    build.build()
    import hyper_connections_stream_b200._lib as L
    L.lib()
    L.set_path({"auto": L.PATH_AUTO, "pipelined": L.PATH_PIPELINED,
                "register": L.PATH_REGISTER}[request.param])
    yield L
    torch.cuda.synchronize()
    assert L.device_fault() == 0
    L.set_path(L.PATH_AUTO)


def _case(T, n, d, R, dt, logits, per_token, seed):
    parts = [gen.to_storage(gen.normal(seed + r, (T, d)), dt) for r in range(R)]
    H = gen.to_storage(gen.normal(seed + 50, (T, n, d)), dt)
    shp = (T, n, n) if per_token else (n, n)
    shv = (T, n) if per_token else (n,)
    if logits:
        A = gen.normal(seed + 51, shp)
        a = gen.normal(seed + 52, shv)
    else:
        A = (np.eye(n, dtype=np.float32) + gen.normal(seed + 51, shp, std=0.05)).astype(np.float32)
        a = gen.normal(seed + 52, shv, mean=1.0 / n, std=0.05)
    b = gen.normal(seed + 53, shv, mean=1.0, std=0.05)
    g = gen.uniform(seed + 54, (d,), 0.5, 1.5)
    return parts, H, A, b, a, g


def _run(hc, parts, H, A, b, a, g, dt, logits, K=20, want_y=True, inplace=False):
    T, n, d = H.shape
    dparts = [to_dev(p, dt) for p in parts]
    dH = to_dev(H, dt)
    y_out = torch.empty((T, d), dtype=TORCH_DT[dt], device="cuda") if want_y else None
    Hp, x = hc.reduce_write_then_read(
        dparts, dH, f32_dev(A), f32_dev(b), f32_dev(a), f32_dev(g), eps=EPS,
        mix=hc.MIX_SINKHORN_LOGITS if logits else hc.MIX_MATRIX, K=K,
        read=hc.READ_SOFTMAX_LOGITS if logits else hc.READ_WEIGHTS,
        out=dH if inplace else None, y_out=y_out)
    torch.cuda.synchronize()
    return (to_host(Hp, dt), to_host(x, dt),
            None if y_out is None else to_host(y_out, dt))


@pytest.mark.parametrize("T,n,d,R,dt,per_token", [
    (37, 4, 1024, 1, "f32", False),
    (64, 4, 7168, 8, "bf16", True),
    (129, 1, 520, 3, "bf16", False),
    (50, 8, 1032, 2, "bf16", True),
    (300, 3, 2056, 5, "f32", True),
    (1, 5, 264, 7, "bf16", False),
    # n <= 2 at widths where the pipelined kernel takes eight-warp groups
    (300, 2, 4096, 8, "bf16", True),
    (77, 1, 4096, 3, "f32", False),
])
def test_static_parameters_bitwise(hc, T, n, d, R, dt, per_token):
    parts, H, A, b, a, g = _case(T, n, d, R, dt, False, per_token, seed=3000 + 7 * T + R)
    Hp, x, y = _run(hc, parts, H, A, b, a, g, dt, logits=False)
    Hr, xr, yr = oracle.reduce_write_then_read(parts, H, A, b, a, g, EPS, dt)
    assert np.array_equal(y, yr)
    assert np.array_equal(Hp, Hr)
    assert np.array_equal(x, xr)


@pytest.mark.parametrize("T,n,d,R,dt", [
    (300, 4, 7168, 8, "bf16"),
    (97, 2, 1544, 4, "bf16"),
    (41, 4, 1024, 3, "f32"),
    (33, 8, 512, 2, "bf16"),
])
def test_logit_parameters(hc, T, n, d, R, dt):
    parts, H, A, b, a, g = _case(T, n, d, R, dt, True, True, seed=3100 + T + R)
    Hp, x, y = _run(hc, parts, H, A, b, a, g, dt, logits=True)
    Hr, xr, yr = oracle.reduce_write_then_read(parts, H, A, b, a, g, EPS, dt, K=20,
                                               mix_logits=True, read_logits=True)
    assert np.array_equal(y, yr)
    assert_close(Hp, Hr, dt, "H'", token_axes=2)
    assert_close(x, xr, dt, "x_next")
    if dt == "bf16":  # fp32 storage keeps the ulp differences of A in every element
        assert np.mean(Hp == Hr) > 0.999


def test_in_place_and_without_y_out(hc):
    parts, H, A, b, a, g = _case(200, 4, 2048, 4, "bf16", False, True, seed=3200)
    Hp, x, y = _run(hc, parts, H, A, b, a, g, "bf16", logits=False, want_y=False, inplace=True)
    Hr, xr, _ = oracle.reduce_write_then_read(parts, H, A, b, a, g, EPS, "bf16")
    assert y is None
    assert np.array_equal(Hp, Hr) and np.array_equal(x, xr)


def test_equals_the_fused_step_on_the_reduced_y(hc):
    """The fused call on R partials gives the bits of hc_write_then_read on
    the oracle's reduced y (the same step after the same reduction)."""
    T, n, d, R, dt = 256, 4, 7168, 8, "bf16"
    parts, H, A, b, a, g = _case(T, n, d, R, dt, True, True, seed=3300)
    Hp, x, y = _run(hc, parts, H, A, b, a, g, dt, logits=True)
    yr = oracle.reduce_partials(parts, dt)
    H2, x2 = hc.write_then_read(to_dev(H, dt), to_dev(yr, dt), f32_dev(A), f32_dev(b), f32_dev(a),
                                f32_dev(g), eps=EPS, mix=hc.MIX_SINKHORN_LOGITS, K=20,
                                read=hc.READ_SOFTMAX_LOGITS)
    torch.cuda.synchronize()
    assert np.array_equal(y, yr)
    assert np.array_equal(Hp, to_host(H2, dt)) and np.array_equal(x, to_host(x2, dt))


def test_full_size_sampled(hc):
    """T = 16384, n = 4, d = 7168, bf16, R = 8, per-token Sinkhorn and softmax
    logits: sampled tokens against the oracle."""
    T, n, d, R, dt = 16384, 4, 7168, 8, "bf16"
    dev = torch.device("cuda")
    parts = [gen.device_normal(3400 + r, (T, d), torch.bfloat16, dev) for r in range(R)]
    H = gen.device_normal(3410, (T, n, d), torch.bfloat16, dev)
    L = gen.device_normal(3411, (T, n, n), torch.float32, dev)
    l = gen.device_normal(3412, (T, n), torch.float32, dev)
    b = torch.from_numpy(gen.normal(3413, (n,), mean=1.0, std=0.02)).to(dev)
    g = torch.ones(d, device=dev)
    y_out = torch.empty((T, d), dtype=torch.bfloat16, device=dev)
    Hp, x = hc.reduce_write_then_read(parts, H, L, b, l, g, eps=EPS, mix=hc.MIX_SINKHORN_LOGITS,
                                      K=20, read=hc.READ_SOFTMAX_LOGITS, y_out=y_out)
    torch.cuda.synchronize()
    rng = np.random.default_rng(23)
    idx = np.unique(np.concatenate([[0, T - 1], rng.choice(T, 126, replace=False)]))
    it = torch.from_numpy(idx).to(dev)
    Hr, xr, yr = oracle.reduce_write_then_read(
        [to_host(p[it], dt) for p in parts], to_host(H[it], dt), L[it].cpu().numpy(),
        b.cpu().numpy(), l[it].cpu().numpy(), g.cpu().numpy(), EPS, dt, K=20, mix_logits=True,
        read_logits=True)
    assert np.array_equal(to_host(y_out[it], dt), yr)
    Hs = to_host(Hp[it], dt)
    assert_close(Hs, Hr, dt, "H'", token_axes=2)
    assert_close(to_host(x[it], dt), xr, dt, "x_next")
    assert np.mean(Hs == Hr) > 0.999


class _Managed:
    """A [T, d] buffer in CUDA managed memory (device-accessible, but not
    device memory of this GPU, so the library reads it with plain loads)."""

    def __init__(self, src: torch.Tensor):
        from cuda.bindings import runtime as rt
        self._rt = rt
        self.bytes = src.numel() * src.element_size()
        err, self.ptr = rt.cudaMallocManaged(self.bytes, rt.cudaMemAttachGlobal)
        assert err == rt.cudaError_t.cudaSuccess, err
        torch.cuda.synchronize()
        err, = rt.cudaMemcpy(self.ptr, src.data_ptr(), self.bytes, rt.cudaMemcpyKind.cudaMemcpyDefault)
        assert err == rt.cudaError_t.cudaSuccess, err

    def free(self):
        torch.cuda.synchronize()
        err, = self._rt.cudaFree(self.ptr)
        assert err == self._rt.cudaError_t.cudaSuccess, err


@pytest.mark.parametrize("T,n,d,R,dt,logits,managed", [
    (600, 4, 7168, 8, "bf16", True, (1, 4, 7)),
    (400, 2, 2048, 3, "f32", False, (0,)),
    (700, 8, 1032, 5, "bf16", False, (0, 1, 2, 3, 4)),
])
def test_partials_read_with_plain_loads(hc, T, n, d, R, dt, logits, managed):
    """Partials outside this GPU's device memory (here managed memory, as a
    peer mapping would be) take the consumers' plain-load branch, in rank
    order with the staged ones: same bits as the oracle."""
    parts, H, A, b, a, g = _case(T, n, d, R, dt, logits, True, seed=3600 + T + R)
    dparts = [to_dev(p, dt) for p in parts]
    held = {r: _Managed(dparts[r]) for r in managed}
    try:
        mixed = [held[r].ptr if r in held else dparts[r] for r in range(R)]
        y_out = torch.empty((T, d), dtype=TORCH_DT[dt], device="cuda")
        Hp, x = hc.reduce_write_then_read(
            mixed, to_dev(H, dt), f32_dev(A), f32_dev(b), f32_dev(a), f32_dev(g), eps=EPS,
            mix=hc.MIX_SINKHORN_LOGITS if logits else hc.MIX_MATRIX, K=20,
            read=hc.READ_SOFTMAX_LOGITS if logits else hc.READ_WEIGHTS, y_out=y_out)
        torch.cuda.synchronize()
    finally:
        for m in held.values():
            m.free()
    Hr, xr, yr = oracle.reduce_write_then_read(parts, H, A, b, a, g, EPS, dt, K=20,
                                               mix_logits=logits, read_logits=logits)
    assert np.array_equal(to_host(y_out, dt), yr)
    if logits:
        assert_close(to_host(Hp, dt), Hr, dt, "H'", token_axes=2)
        assert_close(to_host(x, dt), xr, dt, "x_next")
    else:
        assert np.array_equal(to_host(Hp, dt), Hr) and np.array_equal(to_host(x, dt), xr)


def test_rejections(hc):
    dev = torch.device("cuda")
    T, n, d = 8, 4, 64
    H = torch.zeros((T, n, d), dtype=torch.bfloat16, device=dev)
    y = torch.zeros((T, d), dtype=torch.bfloat16, device=dev)
    A, b, a = torch.eye(n, device=dev), torch.ones(n, device=dev), torch.ones(n, device=dev) / n
    with pytest.raises(ValueError):
        hc.reduce_write_then_read([], H, A, b, a)
    with pytest.raises(ValueError):
        hc.reduce_write_then_read([y] * 9, H, A, b, a)
    with pytest.raises(hc.HCError) as e:   # an output overlapping a partial
        hc.reduce_write_then_read([y, y], H, A, b, a, x_next=y)
    assert e.value.status == hc.HC_ERR_ALIAS
    Hp, x = hc.reduce_write_then_read([y[:0]], H[:0], A, b, a)
    assert Hp.shape == (0, n, d) and x.shape == (0, d)


def _shard(T, r, R):
    base, extra = divmod(T, R)
    return r * base + min(r, extra), base + (1 if r < extra else 0)


@pytest.mark.parametrize("T,n,d,R,dt,logits", [
    (37, 4, 1024, 4, "bf16", False),   # ragged shards: 37 = 4 x 9 + 1
    (300, 4, 7168, 8, "bf16", True),
    (5, 2, 520, 8, "bf16", False),     # fewer tokens than ranks: three ranks own none
    (64, 3, 1032, 3, "f32", False),
    (41, 8, 512, 2, "bf16", True),
])
def test_reduce_scatter_form(hc, T, n, d, R, dt, logits):
    """R ranks emulated on one GPU, one launch per rank: each reduces its
    token shard of the partials, writes its shard of H', and stores its rows
    of x_next into all R x buffers (which start as NaN, so every row must be
    written by exactly one rank). Shards concatenated equal the oracle's step
    over all tokens; every x buffer equals the oracle's x_next."""
    parts, H, A, b, a, g = _case(T, n, d, R, dt, logits, True, seed=3500 + T + R)
    Hr, xr, yr = oracle.reduce_write_then_read(parts, H, A, b, a, g, EPS, dt, K=20,
                                               mix_logits=logits, read_logits=logits)
    sdt = TORCH_DT[dt]
    dparts = [to_dev(p, dt) for p in parts]
    xs = [torch.full((T, d), float("nan"), dtype=sdt, device="cuda") for _ in range(R)]
    Hs, ys = [], []
    for r in range(R):
        t0, Tr = _shard(T, r, R)
        sl = slice(t0, t0 + Tr)
        y_out = torch.empty((Tr, d), dtype=sdt, device="cuda")
        Hs.append(hc.reduce_scatter_write_then_read(
            dparts, xs, r, to_dev(H[sl], dt), f32_dev(A[sl]), f32_dev(b[sl]), f32_dev(a[sl]),
            f32_dev(g), eps=EPS, mix=hc.MIX_SINKHORN_LOGITS if logits else hc.MIX_MATRIX, K=20,
            read=hc.READ_SOFTMAX_LOGITS if logits else hc.READ_WEIGHTS, y_out=y_out))
        ys.append(y_out)
    torch.cuda.synchronize()
    Hp = np.concatenate([to_host(h, dt) for h in Hs])
    assert np.array_equal(np.concatenate([to_host(y, dt) for y in ys]), yr)
    x0 = to_host(xs[0], dt)
    for q in range(1, R):
        assert np.array_equal(to_host(xs[q], dt), x0)
    if logits:
        assert_close(Hp, Hr, dt, "H'", token_axes=2)
        assert_close(x0, xr, dt, "x_next")
    else:
        assert np.array_equal(Hp, Hr) and np.array_equal(x0, xr)


def test_reduce_scatter_rejections(hc):
    dev = torch.device("cuda")
    T, n, d, R = 8, 4, 64, 2
    parts = [torch.zeros((T, d), dtype=torch.bfloat16, device=dev) for _ in range(R)]
    xs = [torch.zeros((T, d), dtype=torch.bfloat16, device=dev) for _ in range(R)]
    H = torch.zeros((T // R, n, d), dtype=torch.bfloat16, device=dev)
    A, b, a = torch.eye(n, device=dev), torch.ones(n, device=dev), torch.ones(n, device=dev) / n
    with pytest.raises(ValueError):      # H is not this rank's shard
        hc.reduce_scatter_write_then_read(parts, xs, 0, H[:1], A, b, a)
    with pytest.raises(hc.HCError) as e:  # two ranks' x buffers are one
        hc.reduce_scatter_write_then_read(parts, [xs[0], xs[0]], 0, H, A, b, a)
    assert e.value.status == hc.HC_ERR_ALIAS
    with pytest.raises(hc.HCError) as e:  # an x buffer is a partial
        hc.reduce_scatter_write_then_read(parts, [xs[0], parts[1]], 1, H, A, b, a)
    assert e.value.status == hc.HC_ERR_ALIAS
