"""GPU parity of the block's output projection fused with the write mix
(`hc_linear_then_write`) against the CPU oracle.

The projection accumulates in fp32 on the tensor cores in their own order, so
y is checked against the fp64 oracle within the accumulation bound
2e-4 * sum_k |X[t,k] Wo[c,k]| plus one bf16 rounding (2^-8 |y|): a wrong tile,
row or channel mapping errs by O(|y|), far outside it. Given the y the kernel
used (stored through y_out), the write mix is a fixed sequence of fp32 FMAs,
so H' must equal the oracle's write mix of that y bit for bit.
"""
from __future__ import annotations

import numpy as np
import pytest
import torch

import hc_inputs as gen
import oracle
from tests._parity import assert_bitwise, f32_dev, to_dev, to_host, values

pytestmark = pytest.mark.gpu


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


def _check_y(y_bits, X, W):
    y64 = oracle.linear(X, W, "bf16")
    mag = np.abs(values(X, "bf16")) @ np.abs(values(W, "bf16")).T
    err = np.abs(values(y_bits, "bf16") - y64)
    bound = 2e-4 * mag + 2.0 ** -8 * np.abs(y64) + 1e-30
    worst = float(np.max(err / bound))
    assert worst <= 1.0, f"y err / bound = {worst:.3f}"


CASES = [(1, 4, 256, 64), (130, 4, 512, 200), (257, 2, 1000, 136), (300, 8, 264, 128),
         (64, 1, 2048, 512), (129, 3, 768, 1024), (200, 5, 520, 72)]


@pytest.mark.parametrize("T,n,d,k", CASES)
@pytest.mark.parametrize("per_token", [False, True])
def test_linear_then_write_matches_oracle(hc, T, n, d, k, per_token):
    dt = "bf16"
    seed = 900 + T + n + d
    X = gen.to_storage(gen.normal(seed, (T, k)), dt)
    W = gen.to_storage(gen.normal(seed + 1, (d, k), std=1.0 / np.sqrt(k)), dt)
    H = gen.to_storage(gen.normal(seed + 2, (T, n, d)), dt)
    if per_token:
        A = gen.normal(seed + 3, (T, n, n), std=0.5)
        b = gen.normal(seed + 4, (T, n), mean=1.0, std=0.1)
    else:
        A = gen.normal(seed + 3, (n, n), std=0.5)
        b = gen.normal(seed + 4, (n,), mean=1.0, std=0.1)
    y = torch.empty((T, d), dtype=torch.bfloat16, device="cuda")
    Hd = to_dev(H, dt)
    H2 = hc.linear_then_write(to_dev(X, dt), to_dev(W, dt), Hd, f32_dev(A), f32_dev(b), y_out=y)
    yh = to_host(y, dt)
    _check_y(yh, X, W)
    assert_bitwise(to_host(H2, dt), oracle.write_mix(H, yh, A, b, dt), "H' (given the kernel's y)")
    # without y_out the same H'; in place gives the same result too
    H3 = hc.linear_then_write(to_dev(X, dt), to_dev(W, dt), Hd, f32_dev(A), f32_dev(b))
    assert torch.equal(H3, H2)
    hc.linear_then_write(to_dev(X, dt), to_dev(W, dt), Hd, f32_dev(A), f32_dev(b), out=Hd)
    assert torch.equal(Hd, H2)


def test_identity_projection_is_the_plain_write(hc):
    """Wo = I (k = d): y is X exactly, so the fused call equals hc_write_mix of X."""
    T, n, d = 150, 4, 512
    X = gen.to_storage(gen.normal(951, (T, d)), "bf16")
    H = gen.to_storage(gen.normal(952, (T, n, d)), "bf16")
    I = gen.to_storage(np.eye(d, dtype=np.float32), "bf16")
    A = gen.normal(953, (n, n), std=0.5)
    b = gen.normal(954, (n,), mean=1.0, std=0.1)
    H2 = hc.linear_then_write(to_dev(X, "bf16"), to_dev(I, "bf16"), to_dev(H, "bf16"),
                              f32_dev(A), f32_dev(b))
    assert_bitwise(to_host(H2, "bf16"), oracle.write_mix(H, X, A, b, "bf16"), "identity projection")


def test_full_size_sampled(hc):
    """T = 16384, n = 4, d = k = 7168 with per-token Sinkhorn-projected A:
    sampled tokens against the oracle."""
    T, n, d, k = 16384, 4, 7168, 7168
    dev = torch.device("cuda")
    X = gen.device_normal(961, (T, k), torch.bfloat16, dev)
    W = gen.device_normal(962, (d, k), torch.bfloat16, dev, std=1.0 / np.sqrt(k))
    H = gen.device_normal(963, (T, n, d), torch.bfloat16, dev)
    L = gen.device_normal(964, (T, n, n), torch.float32, dev)
    A = hc.sinkhorn(L, 20)
    b = torch.from_numpy(gen.normal(965, (n,), mean=1.0, std=0.02)).to(dev)
    y = torch.empty((T, d), dtype=torch.bfloat16, device=dev)
    H2 = hc.linear_then_write(X, W, H, A, b, y_out=y)
    torch.cuda.synchronize()
    rng = np.random.default_rng(13)
    idx = np.unique(np.concatenate([[0, 127, 128, T - 1], rng.choice(T, 28, replace=False)]))
    it = torch.from_numpy(idx).to(dev)
    Xs, Hs, ys = to_host(X[it], "bf16"), to_host(H[it], "bf16"), to_host(y[it], "bf16")
    _check_y(ys, Xs, to_host(W, "bf16"))
    ref = oracle.write_mix(Hs, ys, A[it].cpu().numpy(), b.cpu().numpy(), "bf16")
    assert_bitwise(to_host(H2[it], "bf16"), ref, "H' (sampled)")


def test_rejections(hc):
    dev = torch.device("cuda")
    X = torch.zeros((8, 64), dtype=torch.bfloat16, device=dev)
    W = torch.zeros((64, 64), dtype=torch.bfloat16, device=dev)
    H = torch.zeros((8, 4, 64), dtype=torch.bfloat16, device=dev)
    A, b = torch.eye(4, device=dev), torch.ones(4, device=dev)
    with pytest.raises(hc.HCError) as e:   # k not a multiple of 8
        hc.linear_then_write(X[:, :60].contiguous(), W[:, :60].contiguous(), H, A, b)
    assert e.value.status == hc.HC_ERR_UNSUPPORTED
    with pytest.raises(hc.HCError) as e:   # y_out inside the streams
        hc.linear_then_write(X, W, H, A, b, y_out=H.view(-1)[: 8 * 64].view(8, 64))
    assert e.value.status == hc.HC_ERR_ALIAS
    with pytest.raises(ValueError):
        hc.linear_then_write(X, W[:32], H, A, b)
