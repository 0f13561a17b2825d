"""hc_write_then_read_backward_noalloc (the backward with its gain-gradient
scratch in the library's static device array) against the workspace form on
two successive calls with different inputs: every output bit for bit equal
(same kernels, same launch shapes, same summation order). Collected last so
that the static scratch is first used after every other test has run."""
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


def test_noalloc_rejects_oversize_and_runs_without_dg(hc):
    dev = torch.device("cuda")
    T, n, d = 1024, 2, 32768  # partials: (SMs x CTAs per SM) x d x 4 bytes > 16 MiB
    H, y, L, b, l, g, dHo, dx = _inputs(1701, T, n, d, dev)
    with pytest.raises(hc.HCError) as e:
        hc.write_then_read_backward_noalloc(H, y, L, b, l, g, dHo, dx, mix=hc.MIX_SINKHORN_LOGITS,
                                            K=20, read=hc.READ_SOFTMAX_LOGITS)
    assert e.value.status == hc.HC_ERR_UNSUPPORTED
    # without a gain there is no gain gradient and no scratch is needed
    got = hc.write_then_read_backward_noalloc(H, y, L, b, l, None, dHo, dx,
                                              mix=hc.MIX_SINKHORN_LOGITS, K=20,
                                              read=hc.READ_SOFTMAX_LOGITS)
    ref = hc.write_then_read_backward(H, y, L, b, l, None, dHo, dx, mix=hc.MIX_SINKHORN_LOGITS,
                                      K=20, read=hc.READ_SOFTMAX_LOGITS)
    for key in ("dH", "dy", "dA", "db", "da"):
        assert torch.equal(got[key], ref[key]), key
