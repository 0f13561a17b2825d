"""hc_write_then_read_backward_noalloc -- the backward for callers that may not
allocate device memory when they call it (runtimes that reserve the GPU's
memory up front in their own pool and have no workspace to lend, loops where
a cudaMalloc and the device synchronisation it can bring are not acceptable)
-- keeps its gain-gradient scratch in the library's static device array.

Checked through the C ABI against the workspace form on two successive calls
with different inputs: every output bit for bit equal (same kernels, same
launch shapes, same summation order; the workspace form is itself compared
with the oracle elsewhere). Collected last, so that a run stopping at the
first failure has run every other test before this one."""
from __future__ import annotations

import numpy as np
import pytest
import torch

import hc_inputs as gen

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


def _inputs(seed, T, n, d, dev):
    H = gen.device_normal(seed, (T, n, d), torch.bfloat16, dev)
    y = gen.device_normal(seed + 1, (T, d), torch.bfloat16, dev)
    L = gen.device_normal(seed + 2, (T, n, n), torch.float32, dev)
    l = gen.device_normal(seed + 3, (T, n), torch.float32, dev)
    b = torch.from_numpy(gen.normal(seed + 4, (n,), mean=1.0, std=0.02)).to(dev)
    g = torch.from_numpy(gen.uniform(seed + 5, (d,), 0.5, 1.5)).to(dev)
    dHo = gen.device_normal(seed + 6, (T, n, d), torch.bfloat16, dev)
    dx = gen.device_normal(seed + 7, (T, d), torch.bfloat16, dev)
    return H, y, L, b, l, g, dHo, dx


def test_noalloc_matches_workspace_form_on_two_calls(hc):
    dev = torch.device("cuda")
    T, n, d = 2048, 4, 4096
    for seed in (1501, 1601):
        H, y, L, b, l, g, dHo, dx = _inputs(seed, T, n, d, dev)
        kw = dict(eps=1e-6, mix=hc.MIX_SINKHORN_LOGITS, K=20, read=hc.READ_SOFTMAX_LOGITS)
        ref = hc.write_then_read_backward(H, y, L, b, l, g, dHo, dx, **kw)
        got = hc.write_then_read_backward_noalloc(H, y, L, b, l, g, dHo, dx, **kw)
        torch.cuda.synchronize()
        for key in ("dH", "dy", "dA", "db", "da", "dg"):
            assert torch.equal(got[key], ref[key]), (seed, key)


def test_noalloc_matches_workspace_form_fp32_matrix_weights(hc):
    """fp32 storage, the mixing matrix and read weights given (no Sinkhorn, no
    softmax), per-layer parameters: two calls in a row, bit for bit."""
    dev = torch.device("cuda")
    T, n, d = 777, 3, 1028
    for seed in (1801, 1901):
        H = gen.device_normal(seed, (T, n, d), torch.float32, dev)
        y = gen.device_normal(seed + 1, (T, d), torch.float32, dev)
        A = torch.from_numpy(np.eye(n, dtype=np.float32) + gen.normal(seed + 2, (n, n), std=0.05)).to(dev)
        a = torch.from_numpy(gen.normal(seed + 3, (n,), mean=1.0 / n, std=0.05)).to(dev)
        b = torch.from_numpy(gen.normal(seed + 4, (n,), mean=1.0, std=0.02)).to(dev)
        g = torch.from_numpy(gen.uniform(seed + 5, (d,), 0.5, 1.5)).to(dev)
        dHo = gen.device_normal(seed + 6, (T, n, d), torch.float32, dev)
        dx = gen.device_normal(seed + 7, (T, d), torch.float32, dev)
        ref = hc.write_then_read_backward(H, y, A, b, a, g, dHo, dx, mix=hc.MIX_MATRIX,
                                          read=hc.READ_WEIGHTS)
        got = hc.write_then_read_backward_noalloc(H, y, A, b, a, g, dHo, dx, mix=hc.MIX_MATRIX,
                                                  read=hc.READ_WEIGHTS)
        torch.cuda.synchronize()
        for key in ("dH", "dy", "dA", "db", "da", "dg"):
            assert torch.equal(got[key], ref[key]), (seed, key)


def test_noalloc_no_tokens_is_a_no_op(hc):
    dev = torch.device("cuda")
    n, d = 4, 1024
    H, y, L, b, l, g, dHo, dx = _inputs(2001, 1, n, d, dev)
    got = hc.write_then_read_backward_noalloc(H[:0], y[:0], L[:0], b, l[:0], g, dHo[:0], dx[:0],
                                              mix=hc.MIX_SINKHORN_LOGITS, K=20,
                                              read=hc.READ_SOFTMAX_LOGITS)
    assert got["dH"].shape == (0, n, d) and got["dg"].shape == (d,)


def test_noalloc_rejects_oversize_and_runs_without_dg(hc):
    dev = torch.device("cuda")
    T, n, d = 1024, 2, 32768
    need = int(hc.lib().hc_write_then_read_backward_workspace_bytes(hc._DT[torch.bfloat16], T, n, d))
    assert need > 16 << 20  # the partials alone exceed the static scratch
    H, y, L, b, l, g, dHo, dx = _inputs(1701, T, n, d, dev)
    with pytest.raises(hc.HCError) as e:
        hc.write_then_read_backward_noalloc(H, y, L, b, l, g, dHo, dx, mix=hc.MIX_SINKHORN_LOGITS,
                                            K=20, read=hc.READ_SOFTMAX_LOGITS)
    assert e.value.status == hc.HC_ERR_UNSUPPORTED
    assert "16 MiB" in str(e.value)
    # the workspace form accepts the same call, so the size limit is what refused it
    ref = hc.write_then_read_backward(H, y, L, b, l, g, dHo, dx, mix=hc.MIX_SINKHORN_LOGITS, K=20,
                                      read=hc.READ_SOFTMAX_LOGITS)
    torch.cuda.synchronize()
    assert ref["dg"].shape == (d,)
    # without a gain there is no gain gradient and no scratch is needed
    got = hc.write_then_read_backward_noalloc(H, y, L, b, l, None, dHo, dx,
                                              mix=hc.MIX_SINKHORN_LOGITS, K=20,
                                              read=hc.READ_SOFTMAX_LOGITS)
    ref = hc.write_then_read_backward(H, y, L, b, l, None, dHo, dx, mix=hc.MIX_SINKHORN_LOGITS,
                                      K=20, read=hc.READ_SOFTMAX_LOGITS)
    for key in ("dH", "dy", "dA", "db", "da"):
        assert torch.equal(got[key], ref[key]), key
