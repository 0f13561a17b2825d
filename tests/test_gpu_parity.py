"""GPU parity: the CUDA path (through the C ABI) against the CPU oracle on the
same seeded inputs.

Bar: bit-exact where the arithmetic sequence is fixed on both sides (static
mixing parameters: fp32 FMA chains, fp64 statistic, one storage rounding);
bit-exact on the identity initialisation and on Sinkhorn iteration count and
indexing (0/1 patterns, where exp is exact); otherwise within 1e-5 (fp32
storage) or 2e-2 (bf16 storage) relative error with an rms floor. Large
configurations are checked on a seeded sample of tokens (tokens are
independent), with inputs drawn on the device by torch's generator.
"""
from __future__ import annotations

import numpy as np
import pytest
import torch

import hc_inputs as gen
import oracle
from tests._parity import (RTOL, TORCH_DT, assert_bitwise, assert_close, f32_dev, rel_err,
                           to_dev, to_host, values)

pytestmark = pytest.mark.gpu

EPS = 1e-6


@pytest.fixture(scope="module", params=["auto", "pipelined", "register"])
def hc(request):
    """The binding, with the kernel family chosen automatically (by call size)
    or forced to the pipelined or the register-streaming kernels. After each
    family's tests no kernel may have given up on a bounded wait."""
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


# ---------------------------------------------------------------------------
# Config: tiny correctness, T=256 n=4 d=1024 fp32
# ---------------------------------------------------------------------------

def test_tiny_fp32_static_read_write_fused_bitwise(hc):
    T, n, d, dt, cfg = 256, 4, 1024, "f32", 1
    H = gen.streams(cfg, T, n, d, dt)
    a, A, b = gen.static_params(cfg, n)
    g = np.ones(d, np.float32)
    # read (block input) -> block (harness: tanh) -> fused write + next read
    x_ref = oracle.read_rmsnorm(H, a, g, EPS, dt)
    x_gpu = to_host(hc.read_rmsnorm(to_dev(H, dt), f32_dev(a), f32_dev(g), eps=EPS), dt)
    assert_bitwise(x_gpu, x_ref, "read_rmsnorm")
    y = oracle.block_tanh(x_ref, dt)
    a2, A2, b2 = gen.static_params(cfg, n, layer=1)
    Hw_ref = oracle.write_mix(H, y, A, b, dt)
    Hw_gpu = to_host(hc.write_mix(to_dev(H, dt), to_dev(y, dt), f32_dev(A), f32_dev(b)), dt)
    assert_bitwise(Hw_gpu, Hw_ref, "write_mix")
    H2_ref, x2_ref = oracle.write_then_read(H, y, A, b, a2, g, EPS, dt)
    H2, x2 = hc.write_then_read(to_dev(H, dt), to_dev(y, dt), f32_dev(A), f32_dev(b),
                                f32_dev(a2), f32_dev(g), eps=EPS)
    assert_bitwise(to_host(H2, dt), H2_ref, "fused H'")
    assert_bitwise(to_host(x2, dt), x2_ref, "fused x")


@pytest.mark.parametrize("dt", ["f32", "bf16"])
def test_identity_init_bitwise_and_equal_to_single_stream(hc, dt):
    """a = e_0, A = I, b = 1 with the streams copies of one: GPU equals the
    oracle bit for bit, all streams stay equal, and the result is the
    one-stream pre-norm residual x + tanh(RMSNorm(x) g)."""
    T, n, d, cfg = 256, 4, 1024, 1
    H = gen.copied_streams(cfg, T, n, d, dt)
    a, A, b = gen.identity_params(n)
    g0, g1 = gen.gain(cfg, d, 0), gen.gain(cfg, d, 1)
    x = to_host(hc.read_rmsnorm(to_dev(H, dt), f32_dev(a), f32_dev(g0), eps=EPS), dt)
    assert_bitwise(x, oracle.read_rmsnorm(H, a, g0, EPS, dt), "identity read")
    y = oracle.block_tanh(x, dt)
    H1, x1 = hc.write_then_read(to_dev(H, dt), to_dev(y, dt), f32_dev(A), f32_dev(b),
                                f32_dev(a), f32_dev(g1), eps=EPS)
    H1, x1 = to_host(H1, dt), to_host(x1, dt)
    H1_ref, x1_ref = oracle.write_then_read(H, y, A, b, a, g1, EPS, dt)
    assert_bitwise(H1, H1_ref, "identity H'")
    assert_bitwise(x1, x1_ref, "identity x")
    single = oracle.single_stream_layer(H[:, 0], g0, EPS, dt)
    for j in range(n):
        assert_bitwise(H1[:, j], single, f"stream {j} vs one-stream layer")


# ---------------------------------------------------------------------------
# Config: static HC layer, T=4096 n=4 d=4096 bf16 (unfused and fused)
# ---------------------------------------------------------------------------

def test_static_layer_bf16_unfused_and_fused(hc):
    T, n, d, dt, cfg = 4096, 4, 4096, "bf16", 2
    H = gen.streams(cfg, T, n, d, dt)
    y = gen.block_out(cfg, T, d, dt)
    a, A, b = gen.static_params(cfg, n)
    a2, _, _ = gen.static_params(cfg, n, layer=1)
    g = np.ones(d, np.float32)
    Hd, yd = to_dev(H, dt), to_dev(y, dt)
    x = to_host(hc.read_rmsnorm(Hd, f32_dev(a), f32_dev(g), eps=EPS), dt)
    assert_bitwise(x, oracle.read_rmsnorm(H, a, g, EPS, dt), "read")
    Hw_ref = oracle.write_mix(H, y, A, b, dt)
    Hw = to_host(hc.write_mix(Hd, yd, f32_dev(A), f32_dev(b)), dt)
    assert_bitwise(Hw, Hw_ref, "write")
    xr_ref = oracle.read_rmsnorm(Hw_ref, a2, g, EPS, dt)
    H2, x2 = hc.write_then_read(Hd, yd, f32_dev(A), f32_dev(b), f32_dev(a2), f32_dev(g), eps=EPS)
    assert_bitwise(to_host(H2, dt), Hw_ref, "fused H'")
    assert_bitwise(to_host(x2, dt), xr_ref, "fused x (== unfused write then read)")


# ---------------------------------------------------------------------------
# Config: mHC per-token Sinkhorn, T=16384 n=4 d=7168 bf16, fused
# ---------------------------------------------------------------------------

def _sample_tokens(T, k, seed=5):
    rng = np.random.default_rng(seed)
    idx = np.unique(np.concatenate([[0, T - 1], rng.choice(T, size=min(k, T), replace=False)]))
    return idx


def _mhc_case(hc, T, n, d, dt="bf16", cfg=3, K=20, sample=256, inplace=False):
    dev = torch.device("cuda")
    sdt = TORCH_DT[dt]
    H = gen.device_normal(gen.SEED_H + cfg, (T, n, d), sdt, dev)
    y = gen.device_normal(gen.SEED_Y + cfg, (T, d), sdt, dev)
    L = gen.device_normal(gen.SEED_L + cfg, (T, n, n), torch.float32, dev)
    rl = gen.device_normal(gen.SEED_L + 100 + cfg, (T, n), torch.float32, dev)
    _, _, b = gen.static_params(cfg, n)
    g = np.ones(d, np.float32)
    idx = _sample_tokens(T, sample)
    it = torch.from_numpy(idx).to(dev)
    H_s = to_host(H[it], dt)
    y_s = to_host(y[it], dt)
    L_s = L[it].cpu().numpy()
    rl_s = rl[it].cpu().numpy()
    out = H if inplace else None
    H2, x2 = hc.write_then_read(H, y, L, f32_dev(b), rl, f32_dev(g), eps=EPS,
                                mix=hc.MIX_SINKHORN_LOGITS, K=K, read=hc.READ_SOFTMAX_LOGITS,
                                out=out)
    torch.cuda.synchronize()
    H2_s, x2_s = to_host(H2[it], dt), to_host(x2[it], dt)
    H_ref, x_ref = oracle.write_then_read(H_s, y_s, L_s, b, rl_s, g, EPS, dt, K=K,
                                          mix_logits=True, read_logits=True)
    eH = assert_close(H2_s, H_ref, dt, "mHC H'", token_axes=2)
    ex = assert_close(x2_s, x_ref, dt, "mHC x")
    exact = np.mean(H2_s == H_ref)
    return eH, ex, exact


def test_mhc_sinkhorn_fused_full_size_sampled(hc):
    eH, ex, exact = _mhc_case(hc, 16384, 4, 7168)
    # exp differs by ulps between libm and CUDA; the stored bf16 agrees almost everywhere
    assert exact > 0.999, exact


def test_mhc_fused_in_place(hc):
    eH, ex, exact = _mhc_case(hc, 1024, 4, 7168, inplace=True)
    assert exact > 0.999


def test_sinkhorn_standalone_matches_oracle(hc):
    T, n, K = 16384, 4, 20
    L = gen.mix_logits(3, T, n)
    A = hc.sinkhorn(f32_dev(L), K).cpu().numpy()
    ref = oracle.sinkhorn(L, K)
    err = np.max(np.abs(A.astype(np.float64) - ref) / np.maximum(ref, 1e-30))
    assert err < 1e-5, err
    assert np.max(np.abs(A.astype(np.float64).sum(-2) - 1.0)) <= 1e-6


@pytest.mark.parametrize("n", [1, 2, 3, 4, 5, 8])
def test_sinkhorn_iteration_count_and_indexing_bitwise(hc, n):
    """Logits of 0 and -inf make exp exact (1 and 0), so the GPU and the
    oracle run the same IEEE sums and divisions: equal bit for bit at every K,
    which fixes the pass order, the indexing and the iteration count."""
    rng = np.random.default_rng(100 + n)
    T = 512
    mask = rng.random((T, n, n)) < 0.6
    idx = np.arange(n)
    mask[:, idx, idx] = True                     # every row and column has a 1
    mask[:, idx, (idx + 1) % n] |= rng.random((T, n)) < 0.5
    L = np.where(mask, 0.0, -np.inf).astype(np.float32)
    for K in (1, 2, 3, 7, 20):
        A = hc.sinkhorn(f32_dev(L), K).cpu().numpy()
        assert_bitwise(A, oracle.sinkhorn(L, K), f"n={n} K={K}")
    # K is not off by one: random logits agree with oracle(K) far better than K +- 1
    Lr = gen.normal(200 + n, (T, n, n))
    A = hc.sinkhorn(f32_dev(Lr), 5).cpu().numpy().astype(np.float64)
    if n > 1:
        e5 = np.max(np.abs(A - oracle.sinkhorn(Lr, 5)))
        e4 = np.max(np.abs(A - oracle.sinkhorn(Lr, 4)))
        e6 = np.max(np.abs(A - oracle.sinkhorn(Lr, 6)))
        assert e5 < 1e-6 and e4 > 100 * e5 and e6 > 100 * e5, (e4, e5, e6)


def test_fused_sinkhorn_bitwise_on_exact_logits(hc):
    """The Sinkhorn fused into the write mix, on 0/-inf logits and given read
    weights: H' and x bit-exact (the same projected matrix reaches the FMA
    chain)."""
    T, n, d, dt = 512, 4, 1024, "bf16"
    rng = np.random.default_rng(7)
    mask = rng.random((T, n, n)) < 0.5
    mask[:, np.arange(n), np.arange(n)] = True
    L = np.where(mask, 0.0, -np.inf).astype(np.float32)
    H = gen.streams(9, T, n, d, dt)
    y = gen.block_out(9, T, d, dt)
    a, _, b = gen.static_params(9, n)
    g = gen.gain(9, d)
    H2, x2 = hc.write_then_read(to_dev(H, dt), to_dev(y, dt), f32_dev(L), f32_dev(b), f32_dev(a),
                                f32_dev(g), eps=EPS, mix=hc.MIX_SINKHORN_LOGITS, K=20)
    H_ref, x_ref = oracle.write_then_read(H, y, L, b, a, g, EPS, dt, K=20, mix_logits=True)
    assert_bitwise(to_host(H2, dt), H_ref, "H'")
    assert_bitwise(to_host(x2, dt), x_ref, "x")


# ---------------------------------------------------------------------------
# Config: depth stack, 78 layers, T=8192 n=4 d=7168 bf16, state resident
# ---------------------------------------------------------------------------

def test_depth_stack_78_layers_drift(hc):
    T, n, d, dt, cfg, layers = 8192, 4, 7168, "bf16", 4, 78
    dev = torch.device("cuda")
    sdt = TORCH_DT[dt]
    H = gen.device_normal(gen.SEED_H + cfg, (T, n, d), sdt, dev)
    idx = _sample_tokens(T, 48)
    it = torch.from_numpy(idx).to(dev)
    H_s = to_host(H[it], dt)
    params = [gen.static_params(cfg, n, layer) for layer in range(layers + 1)]
    gains = [gen.gain(cfg, d, layer) for layer in range(layers + 1)]
    P = [(f32_dev(a), f32_dev(A), f32_dev(b)) for (a, A, b) in params]
    Gd = [f32_dev(g) for g in gains]
    # GPU: state stays on the device; block stand-in = torch tanh
    x = hc.read_rmsnorm(H, P[1][0], Gd[1], eps=EPS)
    Hn = torch.empty_like(H)
    for layer in range(1, layers + 1):
        y = torch.tanh(x)
        if layer < layers:
            hc.write_then_read(H, y, P[layer][1], P[layer][2], P[layer + 1][0], Gd[layer + 1],
                               eps=EPS, out=Hn, x_next=x)
        else:
            hc.write_mix(H, y, P[layer][1], P[layer][2], out=Hn)
        H, Hn = Hn, H
    torch.cuda.synchronize()
    H_gpu = to_host(H[it], dt)
    # oracle on the sampled tokens, its own tanh
    Hs = H_s
    xs = oracle.read_rmsnorm(Hs, params[1][0], gains[1], EPS, dt)
    for layer in range(1, layers + 1):
        ys = oracle.block_tanh(xs, dt)
        a_, A_, b_ = params[layer]
        if layer < layers:
            Hs, xs = oracle.write_then_read(Hs, ys, A_, b_, params[layer + 1][0],
                                            gains[layer + 1], EPS, dt)
        else:
            Hs = oracle.write_mix(Hs, ys, A_, b_, dt)
    assert_close(H_gpu, Hs, dt, "depth-78 H", token_axes=2)


# ---------------------------------------------------------------------------
# Config: shape sweep (T x n x d, bf16, per-token Sinkhorn K=20), sampled
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("d", [4096, 7168])
@pytest.mark.parametrize("n", [2, 4, 8])
@pytest.mark.parametrize("T", [1, 64, 1024, 16384, 65536])
def test_shape_sweep_mhc(hc, T, n, d):
    if T * n * d * 2 * 2 > 40e9:
        pytest.skip("beyond this test's memory bound")
    _mhc_case(hc, T, n, d, cfg=5, sample=64, inplace=(T >= 16384))
    torch.cuda.empty_cache()


# ---------------------------------------------------------------------------
# Edge cases
# ---------------------------------------------------------------------------

def test_step_path_reports_the_family_choice(hc):
    """hc_step_path reports the measured per-call choice under automatic
    selection (register-streaming for reads, for writes at n <= 2 and for
    small fused steps; pipelined for the workload's fused step) and the forced
    family otherwise."""
    P, R = hc.PATH_PIPELINED, hc.PATH_REGISTER
    saved = hc.get_path()
    try:
        hc.set_path(hc.PATH_AUTO)
        assert hc.step_path("fused", 16384, 4, 7168) == P
        assert hc.step_path("fused", 64, 4, 7168) == R
        assert hc.step_path("fused", 16384, 1, 4096) == R
        assert hc.step_path("read", 16384, 4, 7168) == R
        assert hc.step_path("read", 65536, 8, 4096) == R
        assert hc.step_path("write", 16384, 2, 7168) == R
        assert hc.step_path("write", 16384, 4, 7168) == P
        assert hc.step_path("write", 64, 4, 7168) == R
        hc.set_path(hc.PATH_PIPELINED)
        assert hc.step_path("read", 64, 4, 7168) == P
        hc.set_path(hc.PATH_REGISTER)
        assert hc.step_path("fused", 16384, 4, 7168) == R
    finally:
        hc.set_path(saved)


@pytest.mark.parametrize("n", [1, 2, 3, 4])
@pytest.mark.parametrize("dt,d", [("bf16", 4096), ("bf16", 2048), ("f32", 4096)])
def test_eight_warp_groups_every_kind(hc, n, dt, d):
    """Widths at which the pipelined family takes eight-warp consumer groups
    (they pad the row's slices less than seven do; read and write kinds up to
    n = 4, the fused step up to n = 2): the read, the write and the fused
    step, bit-exact against the oracle with static parameters, over a ragged
    token count."""
    T = 300
    H = gen.streams(60 + n, T, n, d, dt)
    y = gen.block_out(60 + n, T, d, dt)
    a, A, b = gen.static_params(61 + n, n)
    a2, _, _ = gen.static_params(61 + n, n, layer=1)
    g = gen.gain(62 + n, d)
    Hd, yd = to_dev(H, dt), to_dev(y, dt)
    x = to_host(hc.read_rmsnorm(Hd, f32_dev(a), f32_dev(g), eps=EPS), dt)
    assert_bitwise(x, oracle.read_rmsnorm(H, a, g, EPS, dt), "read")
    Hw_ref = oracle.write_mix(H, y, A, b, dt)
    assert_bitwise(to_host(hc.write_mix(Hd, yd, f32_dev(A), f32_dev(b)), dt), Hw_ref, "write")
    H2, x2 = hc.write_then_read(Hd, yd, f32_dev(A), f32_dev(b), f32_dev(a2), f32_dev(g), eps=EPS)
    assert_bitwise(to_host(H2, dt), Hw_ref, "fused H'")
    assert_bitwise(to_host(x2, dt), oracle.read_rmsnorm(Hw_ref, a2, g, EPS, dt), "fused x")


@pytest.mark.parametrize("n", list(range(1, 9)))
@pytest.mark.parametrize("dt", ["f32", "bf16"])
def test_every_n_ragged_d_per_token_params(hc, n, dt):
    """Every supported n; d that leaves a ragged last slice; per-token A, b, a;
    read weights as logits; a gain vector."""
    T = 37
    d = 8 * 149 if dt == "bf16" else 4 * 149
    H = gen.streams(10 + n, T, n, d, dt)
    y = gen.block_out(10 + n, T, d, dt)
    A = (np.eye(n, dtype=np.float32) + gen.normal(20 + n, (T, n, n), std=0.1)).astype(np.float32)
    b = gen.normal(30 + n, (T, n), mean=1.0, std=0.1)
    rl = gen.normal(40 + n, (T, n))
    g = gen.gain(n, d)
    H2, x2 = hc.write_then_read(to_dev(H, dt), to_dev(y, dt), f32_dev(A), f32_dev(b),
                                f32_dev(rl), f32_dev(g), eps=EPS, read=hc.READ_SOFTMAX_LOGITS)
    H_ref, x_ref = oracle.write_then_read(H, y, A, b, rl, g, EPS, dt, read_logits=True)
    assert_bitwise(to_host(H2, dt), H_ref, "H' (matrix mode is exact)")
    assert_close(to_host(x2, dt), x_ref, dt, "x")
    Hw = hc.write_mix(to_dev(H, dt), to_dev(y, dt), f32_dev(A), f32_dev(b))
    assert_bitwise(to_host(Hw, dt), H_ref, "write_mix")
    xr = hc.read_rmsnorm(to_dev(H, dt), f32_dev(rl), f32_dev(g), eps=EPS,
                         read=hc.READ_SOFTMAX_LOGITS)
    assert_close(to_host(xr, dt), oracle.read_rmsnorm(H, oracle.softmax(rl), g, EPS, dt), dt, "read")


def test_broadcast_logits_and_no_gain(hc):
    """One set of Sinkhorn logits shared by every token (stride 0), g = NULL."""
    T, n, d, dt = 300, 4, 2048, "bf16"
    H = gen.streams(50, T, n, d, dt)
    y = gen.block_out(50, T, d, dt)
    L = gen.normal(51, (n, n))
    b = np.ones(n, np.float32)
    a = np.full(n, 0.25, np.float32)
    H2, x2 = hc.write_then_read(to_dev(H, dt), to_dev(y, dt), f32_dev(L), f32_dev(b), f32_dev(a),
                                None, eps=EPS, mix=hc.MIX_SINKHORN_LOGITS, K=20)
    H_ref, x_ref = oracle.write_then_read(H, y, L, b, a, None, EPS, dt, K=20, mix_logits=True)
    assert_close(to_host(H2, dt), H_ref, dt, "H'", token_axes=2)
    assert_close(to_host(x2, dt), x_ref, dt, "x")


@pytest.mark.parametrize("dt,d", [("bf16", 32768), ("f32", 16384), ("bf16", 9880)])
def test_max_d(hc, dt, d):
    """The largest d each family takes (9880 bf16 is the pipelined limit at n = 4)."""
    T, n = 40, 4
    H = gen.streams(60, T, n, d, dt)
    y = gen.block_out(60, T, d, dt)
    a, A, b = gen.static_params(60, n)
    try:
        H2, x2 = hc.write_then_read(to_dev(H, dt), to_dev(y, dt), f32_dev(A), f32_dev(b),
                                    f32_dev(a), None, eps=EPS)
    except hc.HCError as e:
        if e.status == hc.HC_ERR_UNSUPPORTED and hc.get_path() == hc.PATH_PIPELINED:
            pytest.skip("beyond the pipelined kernels' shared-memory rings")
        raise
    H_ref, x_ref = oracle.write_then_read(H, y, A, b, a, None, EPS, dt)
    assert_bitwise(to_host(H2, dt), H_ref, "H'")
    assert_bitwise(to_host(x2, dt), x_ref, "x")


def test_T_zero_and_T_one(hc):
    dt, n, d = "bf16", 4, 7168
    z = torch.empty((0, n, d), dtype=torch.bfloat16, device="cuda")
    a, A, b = gen.static_params(70, n)
    H2, x2 = hc.write_then_read(z, torch.empty((0, d), dtype=torch.bfloat16, device="cuda"),
                                f32_dev(A), f32_dev(b), f32_dev(a))
    assert H2.shape == (0, n, d) and x2.shape == (0, d)
    _mhc_case(hc, 1, n, d, cfg=70, sample=1)


def test_nan_and_inf_propagate(hc):
    T, n, d, dt = 4, 4, 64, "f32"
    H = gen.streams(80, T, n, d, dt)
    H[1, 2, 5] = np.nan
    H[2, 0, 7] = np.inf
    y = gen.block_out(80, T, d, dt)
    a, A, b = gen.static_params(80, n)
    H2, x2 = hc.write_then_read(to_dev(H, dt), to_dev(y, dt), f32_dev(A), f32_dev(b), f32_dev(a))
    H_ref, x_ref = oracle.write_then_read(H, y, A, b, a, None, EPS, dt)
    g, o = to_host(H2, dt), H_ref
    assert np.array_equal(np.isnan(g), np.isnan(o)) and np.array_equal(np.isinf(g), np.isinf(o))
    fin = np.isfinite(o)
    assert np.array_equal(g[fin], o[fin])
    gx = to_host(x2, dt)
    assert np.array_equal(np.isnan(gx), np.isnan(x_ref))


def test_outputs_stay_inside_their_buffers(hc):
    """Guard regions (canaries) around every output are untouched."""
    T, n, d, dt = 129, 8, 8 * 97, "bf16"
    H = to_dev(gen.streams(90, T, n, d, dt), dt)
    y = to_dev(gen.block_out(90, T, d, dt), dt)
    L = f32_dev(gen.mix_logits(90, T, n))
    rl = f32_dev(gen.read_logits(90, T, n))
    b = f32_dev(np.ones(n, np.float32))
    guard = 4096
    canary = torch.full((guard,), 1234.5, dtype=torch.bfloat16, device="cuda")
    Hbuf = torch.empty(guard * 2 + T * n * d, dtype=torch.bfloat16, device="cuda")
    xbuf = torch.empty(guard * 2 + T * d, dtype=torch.bfloat16, device="cuda")
    for buf in (Hbuf, xbuf):
        buf[:guard] = canary
        buf[-guard:] = canary
    Hout = Hbuf[guard:guard + T * n * d].view(T, n, d)
    x = xbuf[guard:guard + T * d].view(T, d)
    hc.write_then_read(H, y, L, b, rl, None, mix=hc.MIX_SINKHORN_LOGITS, K=20,
                       read=hc.READ_SOFTMAX_LOGITS, out=Hout, x_next=x)
    torch.cuda.synchronize()
    for buf in (Hbuf, xbuf):
        assert torch.equal(buf[:guard], canary) and torch.equal(buf[-guard:], canary)


def test_device_side_argument_errors(hc):
    """Misaligned and partially overlapping device buffers are refused on the
    host before any launch."""
    T, n, d = 16, 4, 1024
    H = torch.zeros((T, n, d), dtype=torch.bfloat16, device="cuda")
    y = torch.zeros((T, d), dtype=torch.bfloat16, device="cuda")
    a, A, b = (f32_dev(v) for v in gen.static_params(1, n))
    L = hc.lib()
    raw = torch.zeros(T * n * d + 64, dtype=torch.bfloat16, device="cuda")
    st = L.hc_write_mix(raw.data_ptr() + 2, y.data_ptr(), H.data_ptr(), hc.HC_BF16, T, n, d, 0,
                        A.data_ptr(), 0, 0, b.data_ptr(), 0, None)
    assert st == hc.HC_ERR_MISALIGNED
    # Hout starts 16 elements into H: partial overlap
    st = L.hc_write_mix(raw.data_ptr(), y.data_ptr(), raw.data_ptr() + 32, hc.HC_BF16, T, n, d,
                        0, A.data_ptr(), 0, 0, b.data_ptr(), 0, None)
    assert st == hc.HC_ERR_ALIAS
    x = torch.zeros((T, d), dtype=torch.bfloat16, device="cuda")
    st = L.hc_write_then_read(H.data_ptr(), y.data_ptr(), H.data_ptr(), H.data_ptr() + 64,
                              hc.HC_BF16, T, n, d, 0, A.data_ptr(), 0, 0, b.data_ptr(), 0, 0,
                              a.data_ptr(), 0, None, 1e-6, None)
    assert st == hc.HC_ERR_ALIAS
    torch.cuda.synchronize()
    assert torch.count_nonzero(x) == 0


def test_bounded_wait_gives_up_and_reports(hc):
    """A wait on a barrier nothing arrives at ends after its limit with fault
    code 32 in the device fault word; the context stays usable."""
    assert hc.device_fault() == 0
    hc.selftest_bounded_wait(2000)
    assert hc.device_fault() == 32
    assert hc.device_fault() == 0  # reading clears it
    # the device still runs the step correctly afterwards
    T, n, d, dt = 8, 4, 1024, "bf16"
    H = gen.streams(3, T, n, d, dt)
    y = gen.block_out(3, T, d, dt)
    a, A, b = gen.static_params(3, n)
    H2, x2 = hc.write_then_read(to_dev(H, dt), to_dev(y, dt), f32_dev(A), f32_dev(b), f32_dev(a))
    H_ref, x_ref = oracle.write_then_read(H, y, A, b, a, None, EPS, dt)
    assert_bitwise(to_host(H2, dt), H_ref, "after self-test")


def test_host_resident_state_matches_device_call(hc):
    """The chunked host-streaming path (copies overlapped with the kernel on
    several streams) gives the same bits as one device call."""
    from hyper_connections_stream_b200 import host
    T, n, d, dt = 1000, 4, 2048, "bf16"
    dev = torch.device("cuda")
    H = gen.device_normal(1011, (T, n, d), torch.bfloat16, dev)
    y = gen.device_normal(2011, (T, d), torch.bfloat16, dev)
    L = gen.device_normal(4011, (T, n, n), torch.float32, dev)
    rl = gen.device_normal(4111, (T, n), torch.float32, dev)
    b = f32_dev(np.ones(n, np.float32))
    g = f32_dev(gen.gain(11, d))
    H2, x2 = hc.write_then_read(H, y, L, b, rl, g, mix=hc.MIX_SINKHORN_LOGITS, K=20,
                                read=hc.READ_SOFTMAX_LOGITS)
    hH, hy, hL, hrl = (t.cpu().pin_memory() for t in (H, y, L, rl))
    oH = torch.empty_like(hH).pin_memory()
    ox = torch.empty((T, d), dtype=torch.bfloat16).pin_memory()
    host.write_then_read_from_host(hH, hy, hL, b, hrl, g, out_H=oH, out_x=ox,
                                   mix=hc.MIX_SINKHORN_LOGITS, K=20,
                                   read=hc.READ_SOFTMAX_LOGITS, chunks=7)
    torch.cuda.synchronize()
    assert torch.equal(oH.view(torch.int16), H2.cpu().view(torch.int16))
    assert torch.equal(ox.view(torch.int16), x2.cpu().view(torch.int16))
