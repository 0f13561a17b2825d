"""GPU parity of the stack ends against the CPU oracle: expansion of one row
into n streams (a bit copy), expansion fused with layer 0's read + RMSNorm,
and the collapse of the n streams by a weighted sum.

Bar: bit-exact for the expansion, for the collapse with weights (one fp32
FMA chain in stream order, one storage rounding) and for the fused read with
static weights (fp64 statistic); within 1e-5 / 2e-2 relative (fp32 / bf16
storage, rms floor) where a softmax of logits sets the weights (exp may differ
by an ulp between the device and the host library).
"""
from __future__ import annotations

import numpy as np
import pytest
import torch

import hc_inputs as gen
import oracle
from tests._parity import assert_bitwise, assert_close, f32_dev, to_dev, to_host

pytestmark = pytest.mark.gpu
EPS = 1e-6


@pytest.fixture(scope="module")
def hc():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from hyper_connections_stream_b200 import build
    build.build()
    import hyper_connections_stream_b200._lib as L
    L.lib()
    yield L
    torch.cuda.synchronize()
    assert L.device_fault() == 0


SHAPES = [(1, 1, 8), (37, 2, 1000), (300, 4, 1024), (129, 3, 2056), (64, 8, 512), (17, 4, 7168)]


@pytest.mark.parametrize("T,n,d", SHAPES)
@pytest.mark.parametrize("dt", ["f32", "bf16"])
def test_expand_bitwise(hc, T, n, d, dt):
    if dt == "f32" and d % 4:
        pytest.skip("fp32 rows are 16-byte vectors")
    x = gen.to_storage(gen.normal(701, (T, d)), dt)
    H = hc.expand(to_dev(x, dt), n)
    assert_bitwise(to_host(H, dt), oracle.expand(x, n, dt), "expand")


@pytest.mark.parametrize("T,n,d", SHAPES)
@pytest.mark.parametrize("dt", ["f32", "bf16"])
def test_expand_then_read_static_bitwise(hc, T, n, d, dt):
    x = gen.to_storage(gen.normal(711, (T, d)), dt)
    a = (np.full(n, 1.0 / n) + gen.normal(712, (n,), std=0.02)).astype(np.float32)
    g = gen.uniform(713, (d,), 0.5, 1.5)
    H_ref, x_ref = oracle.expand_then_read(x, n, a, g, EPS, dt)
    H, xr = hc.expand_then_read(to_dev(x, dt), n, f32_dev(a), f32_dev(g), eps=EPS)
    assert_bitwise(to_host(H, dt), H_ref, "expanded streams")
    assert_bitwise(to_host(xr, dt), x_ref, "layer-0 block input")


@pytest.mark.parametrize("dt", ["f32", "bf16"])
def test_expand_then_read_per_token_logits_and_in_place(hc, dt):
    T, n, d = 333, 4, 2048
    x = gen.to_storage(gen.normal(721, (T, d)), dt)
    l = gen.normal(722, (T, n))
    H_ref, x_ref = oracle.expand_then_read(x, n, l, None, EPS, dt, read_logits=True)
    xd = to_dev(x, dt)
    H, xr = hc.expand_then_read(xd, n, f32_dev(l), None, eps=EPS, read=hc.READ_SOFTMAX_LOGITS,
                                x_read=xd)
    assert xr.data_ptr() == xd.data_ptr()
    assert_bitwise(to_host(H, dt), H_ref, "expanded streams")
    assert_close(to_host(xr, dt), x_ref, dt, "layer-0 block input (logits, in place)")


@pytest.mark.parametrize("T,n,d", SHAPES)
@pytest.mark.parametrize("dt", ["f32", "bf16"])
def test_collapse_weights_bitwise(hc, T, n, d, dt):
    H = gen.to_storage(gen.normal(731, (T, n, d)), dt)
    w = gen.normal(732, (n,))
    wt = gen.normal(733, (T, n))
    out = hc.collapse(to_dev(H, dt), f32_dev(w))
    assert_bitwise(to_host(out, dt), oracle.collapse(H, w, dt), "collapse (shared weights)")
    out = hc.collapse(to_dev(H, dt), f32_dev(wt))
    assert_bitwise(to_host(out, dt), oracle.collapse(H, wt, dt), "collapse (per-token weights)")


@pytest.mark.parametrize("dt", ["f32", "bf16"])
def test_collapse_softmax_logits(hc, dt):
    T, n, d = 257, 4, 4096
    H = gen.to_storage(gen.normal(741, (T, n, d)), dt)
    l = gen.normal(742, (T, n))
    out = hc.collapse(to_dev(H, dt), f32_dev(l), read=hc.READ_SOFTMAX_LOGITS)
    ref = oracle.collapse(H, l, dt, read_logits=True)
    h = to_host(out, dt)
    assert_close(h, ref, dt, "collapse (softmax logits)")
    if dt == "bf16":  # an ulp of a weight rarely survives the bf16 rounding
        assert np.mean(h == ref) > 0.99


def test_full_size_sampled(hc):
    """T = 16384, n = 4, d = 7168 bf16: expand, expand + read, collapse, with
    inputs drawn on the device; checked on sampled tokens."""
    T, n, d, dt = 16384, 4, 7168, "bf16"
    dev = torch.device("cuda")
    x = gen.device_normal(751, (T, d), torch.bfloat16, dev)
    a = torch.full((n,), 0.25, device=dev)
    g = torch.from_numpy(gen.uniform(752, (d,), 0.5, 1.5)).to(dev)
    H, xr = hc.expand_then_read(x, n, a, g, eps=EPS)
    w = torch.from_numpy(gen.normal(753, (n,))).to(dev)
    out = hc.collapse(H, w)
    H2 = hc.expand(x, n)
    torch.cuda.synchronize()
    rng = np.random.default_rng(11)
    idx = np.unique(np.concatenate([[0, T - 1], rng.choice(T, 96, replace=False)]))
    it = torch.from_numpy(idx).to(dev)
    xs = to_host(x[it], dt)
    H_ref, x_ref = oracle.expand_then_read(xs, n, a.cpu().numpy(), g.cpu().numpy(), EPS, dt)
    assert_bitwise(to_host(H[it], dt), H_ref, "expanded (sampled)")
    assert_bitwise(to_host(H2[it], dt), H_ref, "expand only (sampled)")
    assert_bitwise(to_host(xr[it], dt), x_ref, "layer-0 input (sampled)")
    assert_bitwise(to_host(out[it], dt), oracle.collapse(H_ref, w.cpu().numpy(), dt), "collapse")


def test_empty_and_rejections(hc):
    dev = torch.device("cuda")
    x = torch.zeros((0, 64), dtype=torch.bfloat16, device=dev)
    assert hc.expand(x, 4).shape == (0, 4, 64)
    assert hc.collapse(torch.zeros((0, 4, 64), dtype=torch.bfloat16, device=dev),
                       torch.ones(4, device=dev)).shape == (0, 64)
    x = torch.zeros((8, 64), dtype=torch.bfloat16, device=dev)
    buf = torch.zeros(8 * 5 * 64, dtype=torch.bfloat16, device=dev)
    H = buf[: 8 * 4 * 64].view(8, 4, 64)
    with pytest.raises(hc.HCError) as e:   # out overlaps the streams it reads
        hc.collapse(H, torch.ones(4, device=dev), out=buf[8 * 4 * 64 - 64: 8 * 5 * 64 - 64].view(8, 64))
    assert e.value.status == hc.HC_ERR_ALIAS
    with pytest.raises(hc.HCError) as e:   # the copies would overwrite their source
        hc.expand(buf[:8 * 64].view(8, 64), 4, out=H)
    assert e.value.status == hc.HC_ERR_ALIAS
    with pytest.raises(hc.HCError) as e:   # d not a whole number of 16-byte vectors
        hc.expand(torch.zeros((8, 12), dtype=torch.bfloat16, device=dev), 4)
    assert e.value.status == hc.HC_ERR_UNSUPPORTED
    with pytest.raises(ValueError):         # output of the wrong shape never reaches the kernel
        hc.expand(x, 4, out=torch.empty((8, 3, 64), dtype=torch.bfloat16, device=dev))
