"""GPU parity of the input-dependent mixing logits (tcgen05 tensor-core GEMM
with an fp64 RMS statistic) against the fp64 oracle, and of the chain
logits -> Sinkhorn / softmax / write / read against the oracle's chain.

Bound: the tensor cores multiply bf16 x bf16 exactly and accumulate in fp32 in
their own order, so |z - z_ref| <= 2e-4 * r_t * sum_k |u_t[k] W[j][k]| (fp32
accumulation error over n*d terms, with margin) + 1e-6 * |z_ref| (the RMS
factor's rounding). A wrong index, transpose or tile mapping errs by O(1)
relative to that scale.
"""
from __future__ import annotations

import numpy as np
import pytest
import torch

import hc_inputs as gen
import oracle
from tests._parity import assert_close, f32_dev, to_dev, to_host

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
    L.set_path(L.PATH_AUTO)
    yield L
    torch.cuda.synchronize()
    assert L.device_fault() == 0


def _values(bits):
    return (bits.astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def _check_logits(z_gpu, H_bits, W_bits, eps=EPS):
    T, n, d = H_bits.shape
    z_ref = oracle.mix_logits(H_bits, W_bits, eps, "bf16")
    u = _values(H_bits).reshape(T, n * d)
    Wv = _values(W_bits)
    r = 1.0 / np.sqrt(np.mean(u * u, axis=1) + np.float32(eps))
    scale = r[:, None] * (np.abs(u) @ np.abs(Wv).T)
    err = np.abs(z_gpu.astype(np.float64) - z_ref)
    bound = 2e-4 * scale + 1e-6 * np.abs(z_ref)
    worst = np.max(err / np.maximum(bound, 1e-300))
    assert worst <= 1.0, f"logits err/bound = {worst:.3f}"
    return float(np.max(err / np.maximum(scale, 1e-300)))


@pytest.mark.parametrize("T,n,d", [(37, 4, 1024), (300, 2, 4096), (1000, 8, 512),
                                   (5, 4, 1000), (1, 4, 7168), (149, 3, 2048)])
def test_mix_logits_matches_oracle(hc, T, n, d):
    P = n * n + 2 * n
    K = n * d
    H = gen.to_storage(gen.normal(501 + n, (T, n, d)), "bf16")
    W = gen.to_storage(gen.normal(502 + n, (P, K), std=1.0 / np.sqrt(K)), "bf16")
    z = hc.mix_logits(to_dev(H, "bf16"), to_dev(W, "bf16"), eps=EPS).cpu().numpy()
    _check_logits(z, H, W)


def test_mix_logits_full_size_sampled(hc):
    """T = 16384, n = 4, d = 7168 (the mHC workload), checked on sampled tokens."""
    T, n, d = 16384, 4, 7168
    P, K = n * n + 2 * n, n * d
    dev = torch.device("cuda")
    H = gen.device_normal(gen.SEED_H + 3, (T, n, d), torch.bfloat16, dev)
    W = gen.device_normal(503, (P, K), torch.bfloat16, dev, std=1.0 / np.sqrt(K))
    z = hc.mix_logits(H, W, eps=EPS)
    torch.cuda.synchronize()
    rng = np.random.default_rng(9)
    idx = np.unique(np.concatenate([[0, 111, 112, T - 1], rng.choice(T, 120, replace=False)]))
    it = torch.from_numpy(idx).to(dev)
    _check_logits(z[it].cpu().numpy(), to_host(H[it], "bf16"), to_host(W, "bf16"))


def test_mix_logits_one_hot_weights_pick_stream_values(hc):
    """A one-hot weight row returns r_t * u_t[k]: fixes which element each
    output column reads (stream, channel) and the row/token mapping."""
    T, n, d = 260, 4, 512
    K = n * d
    H = gen.to_storage(gen.normal(510, (T, n, d)), "bf16")
    P = 24
    W32 = np.zeros((P, K), np.float32)
    picks = [(j * 331 + 7) % K for j in range(P)]
    for j, k in enumerate(picks):
        W32[j, k] = 1.0
    W = gen.to_storage(W32, "bf16")
    z = hc.mix_logits(to_dev(H, "bf16"), to_dev(W, "bf16"), eps=EPS).cpu().numpy()
    u = _values(H).reshape(T, K)
    r = 1.0 / np.sqrt(np.mean(u * u, axis=1) + np.float32(EPS))
    want = r[:, None] * u[:, picks]
    assert np.max(np.abs(z - want) / (np.abs(want) + 1e-30)) < 1e-5


def test_logits_feed_the_fused_step(hc):
    """logits -> per-token Sinkhorn logits, read logits and write gains (token
    stride P views) -> fused step; against the oracle's own chain."""
    T, n, d, dt = 512, 4, 2048, "bf16"
    P, K = n * n + 2 * n, n * d
    H = gen.to_storage(gen.normal(520, (T, n, d)), dt)
    y = gen.to_storage(gen.normal(521, (T, d)), dt)
    W = gen.to_storage(gen.normal(522, (P, K), std=1.0 / np.sqrt(K)), dt)
    g = gen.gain(520, d)
    Hd = to_dev(H, dt)
    z = hc.mix_logits(Hd, to_dev(W, dt), eps=EPS)
    L = z[:, : n * n].view(T, n, n)
    rl = z[:, n * n: n * n + n]
    b = z[:, n * n + n:]
    H2, x2 = hc.write_then_read(Hd, to_dev(y, dt), L, b, rl, f32_dev(g), eps=EPS,
                                mix=hc.MIX_SINKHORN_LOGITS, K=20, read=hc.READ_SOFTMAX_LOGITS)
    zr = oracle.mix_logits(H, W, EPS, dt).astype(np.float32)
    H_ref, x_ref = oracle.write_then_read(H, y, zr[:, : n * n].reshape(T, n, n),
                                          np.ascontiguousarray(zr[:, n * n + n:]),
                                          np.ascontiguousarray(zr[:, n * n: n * n + n]), g, EPS,
                                          dt, K=20, mix_logits=True, read_logits=True)
    H2h, x2h = to_host(H2, dt), to_host(x2, dt)
    assert_close(H2h, H_ref, dt, "chained H'", token_axes=2)
    assert np.mean(H2h == H_ref) > 0.99
    # The two chains start from logits that agree to fp32 accumulation error,
    # so a stored H' element may differ by one bf16 ulp (at most 2^-7 of its
    # magnitude); through the read mix (which can cancel) that moves x by up to
    # sum_i a_i |H'_i| 2^-7 r g, plus one ulp of x itself. Check against that
    # propagated bound.
    a = oracle.softmax(np.ascontiguousarray(zr[:, n * n: n * n + n])).astype(np.float64)
    Hv = _values(H_ref)                                    # [T, n, d]
    h = np.einsum("ti,tik->tk", a, Hv)
    r = 1.0 / np.sqrt(np.mean(h * h, axis=1) + np.float32(EPS))
    spread = np.einsum("ti,tik->tk", np.abs(a), np.abs(Hv)) * 2.0 ** -7
    xv, xr = _values(x2h), _values(x_ref)
    bound = 1.5 * spread * r[:, None] * g[None, :] + 2.0 ** -7 * np.abs(xr) + 1e-30
    assert np.all(np.abs(xv - xr) <= bound), float(np.max(np.abs(xv - xr) / bound))
    assert np.mean(x2h == x_ref) > 0.99
