"""GPU parity of the backward pass (hc_write_then_read_backward) against the
CPU oracle's fp64 backward on the same inputs.

Both sides recompute the forward with the same fp32 arithmetic; the GPU then
runs the backward in fp32 (fp64 per-token statistics and cross-warp sums, the
Sinkhorn backward in fp32) while the oracle runs it in fp64. Bars: dH and dy
elementwise within 1e-4 (fp32 storage) or 2e-2 (bf16 storage, the outputs are
rounded to bf16) relative with the per-token rms floor; the per-token
parameter gradients and dg within 2e-4 of the tensor's largest magnitude
(fp32 sums of thousands of products, and 40 fp32 Sinkhorn passes undone),
except the read-logit gradient for bf16 storage with logit-mode parameters:
within 1e-3 (DA_BF16_LOGITS). There the exp of the Sinkhorn and softmax
definitions differs by ulps between the two sides, a small fraction of the
recomputed H' rounds to the adjacent bf16 value, and the softmax backward
(a difference of near-equal sums) turns that into up to 2.5e-4 of the largest
magnitude; the oracle's own da moves that much when its logits move by 6e-8
(tests/test_oracle_pins.py::test_backward_read_logit_gradient_conditioning).
A wrong index, transpose or sign errs by O(1) relative to those scales.
"""
from __future__ import annotations

import numpy as np
import pytest
import torch

import hc_inputs as gen
import oracle
from tests._parity import f32_dev, rel_err, to_dev, to_host, values

pytestmark = pytest.mark.gpu
EPS = 1e-6
DA_BF16_LOGITS = 1e-3


def _param_bar(key, dt, mix, read):
    return DA_BF16_LOGITS if (key == "da" and dt == "bf16" and (mix or read)) else 2e-4


@pytest.fixture(scope="module", params=["auto", "pipelined", "register"])
def hc(request):
    """The binding with the backward's step kernel chosen automatically (the
    register kernel), forced to the TMA-fed kernel (bf16, n <= 4; other calls
    keep the register kernel) or forced to the register kernel."""
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


def _inputs(T, n, d, dt, mix, read, per_token, seed, with_dHout=True):
    H = gen.to_storage(gen.normal(seed, (T, n, d)), dt)
    y = gen.to_storage(gen.normal(seed + 1, (T, d)), dt)
    shapeA = (T, n, n) if per_token else (n, n)
    shape_v = (T, n) if per_token else (n,)
    A = gen.normal(seed + 2, shapeA, std=1.0 if mix else 0.5)
    b = gen.normal(seed + 3, shape_v, mean=1.0, std=0.1)
    a = gen.normal(seed + 4, shape_v, std=1.0 if read else 0.5)
    g = gen.uniform(seed + 5, (d,), 0.5, 1.5)
    dHo = gen.to_storage(gen.normal(seed + 6, (T, n, d)), dt) if with_dHout else None
    dx = gen.to_storage(gen.normal(seed + 7, (T, d)), dt)
    return H, y, A, b, a, g, dHo, dx


def _check(hc, T, n, d, dt, mix, read, per_token, seed, with_dHout=True, K=20):
    H, y, A, b, a, g, dHo, dx = _inputs(T, n, d, dt, mix, read, per_token, seed, with_dHout)
    got = hc.write_then_read_backward(
        to_dev(H, dt), to_dev(y, dt), f32_dev(A), f32_dev(b), f32_dev(a), f32_dev(g),
        None if dHo is None else to_dev(dHo, dt), to_dev(dx, dt), eps=EPS,
        mix=hc.MIX_SINKHORN_LOGITS if mix else hc.MIX_MATRIX, K=K,
        read=hc.READ_SOFTMAX_LOGITS if read else hc.READ_WEIGHTS)
    ref = oracle.write_then_read_backward(H, y, A, b, a, g, EPS, dt,
                                          None if dHo is None else values(dHo, dt),
                                          values(dx, dt), K=K, mix_logits=mix, read_logits=read)
    rtol = 1e-4 if dt == "f32" else 2e-2
    for key, axes in (("dH", 2), ("dy", 1)):
        gv = values(to_host(got[key], dt), dt)
        o = ref[key]
        lead = o.shape[:axes]
        o2 = o.reshape(*lead, -1)
        rms = np.sqrt(np.mean(o2 * o2, axis=-1, keepdims=True))
        den = np.maximum(np.abs(o2), rms) + 1e-30
        e = float(np.max(np.abs(gv.reshape(*lead, -1) - o2) / den))
        assert e <= rtol, f"{key}: rel err {e:.3e}"
    for key in ("dA", "db", "da", "dg"):
        gv = got[key].cpu().numpy().astype(np.float64)
        o = ref[key]
        e = float(np.max(np.abs(gv - o)) / (np.max(np.abs(o)) + 1e-30))
        assert e <= _param_bar(key, dt, mix, read), f"{key}: err / max {e:.3e}"


@pytest.mark.parametrize("T,n,d,dt,mix,read,per_token", [
    (37, 4, 1024, "f32", True, True, True),
    (64, 4, 2048, "bf16", True, True, True),
    (50, 2, 512, "f32", False, False, False),
    (33, 8, 512, "bf16", True, True, True),
    (20, 1, 256, "f32", False, True, True),
    (129, 3, 1000, "f32", True, False, True),
    (300, 4, 7168, "bf16", True, True, True),
    (17, 6, 264, "bf16", False, True, False),
    # bf16 at every n <= 5: ragged T and d, one token, and enough tokens per
    # CTA for several parameter batches
    (1, 4, 520, "bf16", True, True, True),
    (41, 1, 1032, "bf16", False, True, True),
    (150, 2, 776, "bf16", True, False, True),
    (97, 3, 1544, "bf16", True, True, False),
    (61, 5, 2056, "bf16", True, True, True),
    (2000, 4, 1024, "bf16", True, True, True),
    # wide rows: h parked without the staging ring (d = 16384), and h rebuilt
    # in phase 2 because even the parked row does not fit (d = 32768)
    (20, 4, 16384, "bf16", True, True, True),
    (9, 2, 32768, "bf16", False, True, True),
    # fp32 beyond n = 4 (two-element vectors, 8-byte staging copies)
    (23, 6, 1000, "f32", True, True, True),
    (19, 8, 520, "f32", True, False, True),
])
def test_backward_matches_oracle(hc, T, n, d, dt, mix, read, per_token):
    _check(hc, T, n, d, dt, mix, read, per_token, seed=1200 + T + n)


def test_backward_bf16_without_dHout(hc):
    _check(hc, 90, 4, 1024, "bf16", True, True, True, seed=1350, with_dHout=False, K=3)


def test_backward_without_dHout_and_small_K(hc):
    _check(hc, 40, 4, 512, "f32", True, True, True, seed=1300, with_dHout=False, K=1)


def test_backward_full_size_sampled(hc):
    """T = 16384, n = 4, d = 7168, bf16, per-token Sinkhorn and softmax logits:
    per-token outputs on sampled tokens against the oracle; dg, a sum over all
    tokens, equals the sum of per-chunk gains computed by the library over the
    same tokens in 8 separate calls (order-independent up to fp32 rounding)."""
    T, n, d, dt = 16384, 4, 7168, "bf16"
    dev = torch.device("cuda")
    H = gen.device_normal(1401, (T, n, d), torch.bfloat16, dev)
    y = gen.device_normal(1402, (T, d), torch.bfloat16, dev)
    L = gen.device_normal(1403, (T, n, n), torch.float32, dev)
    l = gen.device_normal(1404, (T, n), torch.float32, dev)
    b = torch.from_numpy(gen.normal(1405, (n,), mean=1.0, std=0.02)).to(dev)
    g = torch.from_numpy(gen.uniform(1406, (d,), 0.5, 1.5)).to(dev)
    dHo = gen.device_normal(1407, (T, n, d), torch.bfloat16, dev)
    dx = gen.device_normal(1408, (T, d), torch.bfloat16, dev)
    got = hc.write_then_read_backward(H, y, L, b, l, g, dHo, dx, eps=EPS, mix=hc.MIX_SINKHORN_LOGITS,
                                      K=20, read=hc.READ_SOFTMAX_LOGITS)
    torch.cuda.synchronize()
    rng = np.random.default_rng(17)
    idx = np.unique(np.concatenate([[0, T - 1], rng.choice(T, 62, replace=False)]))
    it = torch.from_numpy(idx).to(dev)
    ref = oracle.write_then_read_backward(
        to_host(H[it], dt), to_host(y[it], dt), L[it].cpu().numpy(), b.cpu().numpy(),
        l[it].cpu().numpy(), g.cpu().numpy(), EPS, dt, values(to_host(dHo[it], dt), dt),
        values(to_host(dx[it], dt), dt), K=20, mix_logits=True, read_logits=True, want_dg=False)
    for key in ("dH", "dy"):
        gv = values(to_host(got[key][it], dt), dt)
        o = ref[key].reshape(len(idx), -1)
        rms = np.sqrt(np.mean(o * o, axis=-1, keepdims=True))
        e = float(np.max(np.abs(gv.reshape(len(idx), -1) - o) / np.maximum(np.abs(o), rms)))
        assert e <= 2e-2, (key, e)
    for key in ("dA", "db", "da"):
        gv = got[key][it].cpu().numpy().astype(np.float64)
        e = float(np.max(np.abs(gv - ref[key])) / np.max(np.abs(ref[key])))
        assert e <= _param_bar(key, dt, True, True), (key, e)
    parts = []
    for c in range(8):
        sl = slice(c * T // 8, (c + 1) * T // 8)
        parts.append(hc.write_then_read_backward(H[sl], y[sl], L[sl], b, l[sl], g, dHo[sl], dx[sl],
                                                 eps=EPS, mix=hc.MIX_SINKHORN_LOGITS, K=20,
                                                 read=hc.READ_SOFTMAX_LOGITS)["dg"].double())
    dg_sum = torch.stack(parts).sum(0)
    rel = float((got["dg"].double() - dg_sum).abs().max() / dg_sum.abs().max())
    assert rel < 1e-5, rel


def test_backward_rejections(hc):
    dev = torch.device("cuda")
    T, n, d = 8, 4, 64
    H = torch.zeros((T, n, d), dtype=torch.bfloat16, device=dev)
    y = torch.zeros((T, d), dtype=torch.bfloat16, device=dev)
    A, b, a = torch.zeros((n, n), device=dev), torch.ones(n, device=dev), torch.ones(n, device=dev)
    g = torch.ones(d, device=dev)
    with pytest.raises(hc.HCError) as e:   # workspace too small for dg
        hc.write_then_read_backward(H, y, A, b, a, g, None, y, workspace=torch.empty(
            16, dtype=torch.uint8, device=dev))
    assert e.value.status == hc.HC_ERR_INVALID_ARG
    with pytest.raises(hc.HCError) as e:   # Sinkhorn history does not fit shared memory
        hc.write_then_read_backward(H, y, A, b, a, g, None, y, mix=hc.MIX_SINKHORN_LOGITS, K=5000)
    assert e.value.status == hc.HC_ERR_UNSUPPORTED
    out = hc.write_then_read_backward(H[:0], y[:0], A, b, a, g, None, y[:0])
    assert out["dH"].shape == (0, n, d)
