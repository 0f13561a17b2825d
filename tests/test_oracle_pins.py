"""Pins for the CPU oracle: each test checks the oracle against something that is
not the oracle -- exact rational arithmetic, closed forms, invariants the pages
fix, or a library routine -- so that a plausible mistake in it (a dropped term,
a wrong sign or index, a transposed operand, a reordered Sinkhorn pass, a
misplaced eps) fails at least one test.

Sources: "Hyper-connections (mHC)" glossary entry (hfviewer), definition
paragraph (learned mixing before and after each block; mHC makes it doubly
stochastic with a few Sinkhorn iterations); "Tencent open-sources Hy4 Preview
at 770B -- Identity Hyper-Connections" (learnaivisually), TL;DR and Jargon
(identity initialisation, pre-norm) and "What four streams cost per token".
"""
from __future__ import annotations

import json
import math
import os
from decimal import Decimal, getcontext
from fractions import Fraction

import numpy as np
import pytest
import torch

import hc_inputs as gen
import oracle
from tests._parity import values

U32 = 2.0 ** -24  # unit roundoff of fp32
HERE = os.path.dirname(os.path.abspath(__file__))


def f32_of(bits_or_vals, dt):
    """Storage values -> float64 numpy, through torch (independent of the oracle)."""
    if dt == "f32":
        return np.asarray(bits_or_vals, dtype=np.float32).astype(np.float64)
    t = torch.from_numpy(np.ascontiguousarray(bits_or_vals).view(np.int16)).view(torch.bfloat16)
    return t.to(torch.float64).numpy()


# --------------------------------------------------------------------------
# storage rounding
# --------------------------------------------------------------------------

def test_bf16_rounding_matches_torch():
    rng = np.random.default_rng(7)
    x = rng.standard_normal(20000).astype(np.float32) * np.float32(3.0)
    # exact ties between two bf16 values, both parities of the kept bit
    ties = (np.arange(1, 4001, dtype=np.uint32) << 16 | np.uint32(0x8000)).view(np.float32)
    special = np.array([0.0, -0.0, np.inf, -np.inf, 3.3895314e38, -3.3895314e38,
                        1e-40, -1e-40, 65504.0, 1.0 + 2 ** -8, 1.0 + 3 * 2 ** -9],
                       dtype=np.float32)
    allv = np.concatenate([x, ties, -ties, special])
    got = oracle.round_to(allv, "bf16")
    want = torch.from_numpy(allv).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(got, want)
    nan = oracle.round_to(np.array([np.nan], np.float32), "bf16")
    assert np.isnan(torch.from_numpy(nan.view(np.int16)).view(torch.bfloat16).float().numpy()[0])


# --------------------------------------------------------------------------
# Sinkhorn projection (mHC)
# --------------------------------------------------------------------------

def test_sinkhorn_hand_expanded_n2():
    """exp(L) = [[1,3],[1,1]]; worked by hand in exact fractions.
    K=1: rows -> [[1/4,3/4],[1/2,1/2]], then columns -> [[1/3,3/5],[2/3,2/5]].
    K=2: rows -> [[5/14,9/14],[5/8,3/8]], columns -> [[4/11,12/19],[7/11,7/19]].
    Columns-first would give [[2/5,3/5],[2/3,1/3]] at K=1, so this also pins
    the pass order and that K counts row+column pairs."""
    L = np.array([[0.0, math.log(3.0)], [0.0, 0.0]], np.float32)
    k1 = np.array([[1 / 3, 3 / 5], [2 / 3, 2 / 5]])
    k2 = np.array([[4 / 11, 12 / 19], [7 / 11, 7 / 19]])
    k0 = np.array([[1.0, 3.0], [1.0, 1.0]])
    for K, want in ((0, k0), (1, k1), (2, k2)):
        got32 = oracle.sinkhorn(L, K)
        got64 = oracle.sinkhorn(L.astype(np.float64), K, f64=True)
        assert np.allclose(got32, want, rtol=2e-6, atol=0), (K, got32)
        assert np.allclose(got64, want, rtol=1e-6, atol=0), (K, got64)


@pytest.mark.parametrize("n", [2, 3, 4, 8])
def test_sinkhorn_columns_sum_to_one_at_every_K(n):
    L = gen.normal(11 + n, (512, n, n))
    for K in (1, 2, 3, 5, 10, 20, 25):
        A = oracle.sinkhorn(L, K)
        assert np.all(A > 0)
        assert np.max(np.abs(A.astype(np.float64).sum(axis=-2) - 1.0)) <= 1e-6
        A64 = oracle.sinkhorn(L.astype(np.float64), K, f64=True)
        assert np.max(np.abs(A64.sum(axis=-2) - 1.0)) <= 1e-13


@pytest.mark.parametrize("n", [2, 4, 8])
def test_sinkhorn_rows_converge(n):
    """At K=200 rows sum to 1 within 1e-6 too (the limit is doubly stochastic).
    At K=20 the row residual is not below 1e-6 for every token; on the tokens
    where the fp64 projection already is, the fp32 one is as well."""
    L = gen.normal(21 + n, (2048, n, n))
    A = oracle.sinkhorn(L, 200)
    assert np.max(np.abs(A.astype(np.float64).sum(axis=-1) - 1.0)) <= 1e-6
    A64_20 = oracle.sinkhorn(L.astype(np.float64), 20, f64=True)
    ok = np.max(np.abs(A64_20.sum(axis=-1) - 1.0), axis=-1) <= 1e-7
    assert ok.mean() > 0.5
    A32_20 = oracle.sinkhorn(L, 20)
    assert np.max(np.abs(A32_20[ok].astype(np.float64).sum(axis=-1) - 1.0)) <= 1e-6


def test_sinkhorn_n2_limit_closed_form():
    """A positive 2x2 matrix's Sinkhorn limit is [[p,1-p],[1-p,p]] and the
    diagonal scalings keep the cross ratio, so p/(1-p) = exp(D/2) with
    D = l00 + l11 - l01 - l10."""
    L = gen.normal(31, (256, 2, 2)).astype(np.float64)
    A = oracle.sinkhorn(L, 2000, f64=True)
    D = L[:, 0, 0] + L[:, 1, 1] - L[:, 0, 1] - L[:, 1, 0]
    p = 1.0 / (1.0 + np.exp(-D / 2))
    want = np.stack([np.stack([p, 1 - p], -1), np.stack([1 - p, p], -1)], -2)
    assert np.max(np.abs(A - want)) < 1e-12


@pytest.mark.parametrize("n", [3, 4, 8])
@pytest.mark.parametrize("K", [1, 4, 20])
def test_sinkhorn_cross_ratio_is_that_of_exp_logits(n, K):
    """Row and column passes are diagonal scalings, so at every K
    A[i,j] A[k,l] / (A[i,l] A[k,j]) = exp(L[i,j] + L[k,l] - L[i,l] - L[k,j]).
    A transposed output or a wrong exponent breaks this."""
    L = gen.normal(41 + n, (64, n, n)).astype(np.float64)
    A = oracle.sinkhorn(L, K, f64=True)
    lA = np.log(A)
    for (i, k, j, l) in ((0, 1, 0, 1), (0, n - 1, 1, n - 1), (1, 2, 0, 2)):
        lhs = lA[:, i, j] + lA[:, k, l] - lA[:, i, l] - lA[:, k, j]
        rhs = L[:, i, j] + L[:, k, l] - L[:, i, l] - L[:, k, j]
        assert np.max(np.abs(lhs - rhs)) < 1e-12
    A32 = oracle.sinkhorn(L.astype(np.float32), K).astype(np.float64)
    lA = np.log(A32)
    lhs = lA[:, 0, 0] + lA[:, 1, 1] - lA[:, 0, 1] - lA[:, 1, 0]
    rhs = L[:, 0, 0] + L[:, 1, 1] - L[:, 0, 1] - L[:, 1, 0]
    assert np.max(np.abs(lhs - rhs)) < 2e-5


def test_sinkhorn_row_shift_invariance_and_column_shift_dependence():
    """Adding c to a row of L is undone by the first row pass (any K >= 1);
    adding c to a column is not undone at finite K, only in the limit."""
    L = gen.normal(51, (128, 4, 4)).astype(np.float64)
    base = oracle.sinkhorn(L, 20, f64=True)
    Lr = L.copy(); Lr[:, 2, :] += 1.7
    assert np.max(np.abs(oracle.sinkhorn(Lr, 20, f64=True) - base)) < 1e-14
    Lc = L.copy(); Lc[:, :, 2] += 1.7
    diff = np.max(np.abs(oracle.sinkhorn(Lc, 20, f64=True) - base))
    assert diff > 1e-9
    lim = oracle.sinkhorn(L, 3000, f64=True)
    assert np.max(np.abs(oracle.sinkhorn(Lc, 3000, f64=True) - lim)) < 1e-10


def test_sinkhorn_permutation_equivariance():
    rng = np.random.default_rng(61)
    L = gen.normal(61, (64, 5, 5))
    p = rng.permutation(5); q = rng.permutation(5)
    A = oracle.sinkhorn(L, 20)
    Ap = oracle.sinkhorn(L[:, p][:, :, q], 20)
    assert np.allclose(Ap, A[:, p][:, :, q], rtol=2e-6, atol=1e-7)


def test_sinkhorn_equal_logits_and_n1():
    for n in (2, 3, 4, 8):
        A = oracle.sinkhorn(np.full((3, n, n), 0.37, np.float32), 20)
        assert np.max(np.abs(A.astype(np.float64) - 1.0 / n)) <= 1.0 / n * 2 * U32
    A1 = oracle.sinkhorn(np.array([[[2.5]]], np.float32), 20)
    assert A1.reshape(-1)[0] == 1.0


# --------------------------------------------------------------------------
# read-weight softmax (mHC)
# --------------------------------------------------------------------------

def test_softmax_against_library_and_closed_forms():
    l = gen.normal(71, (1000, 4))
    a = oracle.softmax(l).astype(np.float64)
    ref = torch.softmax(torch.from_numpy(l.astype(np.float64)), dim=-1).numpy()
    assert np.max(np.abs(a - ref)) < 4e-7
    assert np.max(np.abs(a.sum(-1) - 1.0)) < 5e-7
    eq = oracle.softmax(np.full((2, 4), -3.0, np.float32))
    assert np.all(eq == np.float32(0.25))
    l2 = gen.normal(72, (500, 2))
    a2 = oracle.softmax(l2).astype(np.float64)
    sig = 1.0 / (1.0 + np.exp(-(l2[:, 0].astype(np.float64) - l2[:, 1])))
    assert np.max(np.abs(a2[:, 0] - sig)) < 3e-7


# --------------------------------------------------------------------------
# write mix: H'_j = sum_i A[i,j] H_i + b_j y
# --------------------------------------------------------------------------

def test_write_mix_hand_expanded_n2():
    """n = 2 written out term by term: H'_0 = A00 H0 + A10 H1 + b0 y,
    H'_1 = A01 H0 + A11 H1 + b1 y (row of A = source stream)."""
    H = np.array([[[1.0, -2.0, 0.5], [4.0, 0.25, -1.0]]], np.float32)
    y = np.array([[2.0, 8.0, -4.0]], np.float32)
    A = np.array([[0.5, 0.25], [0.125, 2.0]], np.float32)
    b = np.array([1.0, -0.5], np.float32)
    out = oracle.write_mix(H, y, A, b, "f32")
    h0, h1 = H[0, 0].astype(np.float64), H[0, 1].astype(np.float64)
    yy = y[0].astype(np.float64)
    want0 = 0.5 * h0 + 0.125 * h1 + 1.0 * yy
    want1 = 0.25 * h0 + 2.0 * h1 - 0.5 * yy
    assert np.array_equal(out[0, 0], want0.astype(np.float32))  # exact in binary
    assert np.array_equal(out[0, 1], want1.astype(np.float32))


@pytest.mark.parametrize("n", [1, 2, 4])
@pytest.mark.parametrize("dt", ["f32", "bf16"])
def test_write_mix_brute_force_exact_rationals(n, dt):
    d, T = 16, 3
    H = gen.to_storage(gen.normal(81 + n, (T, n, d)), dt)
    y = gen.to_storage(gen.normal(82 + n, (T, d)), dt)
    A = gen.normal(83 + n, (T, n, n))
    b = gen.normal(84 + n, (T, n))
    out = f32_of(oracle.write_mix(H, y, A, b, dt), dt)
    Hv, yv = f32_of(H, dt), f32_of(y, dt)
    for t in range(T):
        for j in range(n):
            for k in range(d):
                terms = [Fraction(float(A[t, i, j])) * Fraction(float(Hv[t, i, k]))
                         for i in range(n)]
                terms.append(Fraction(float(b[t, j])) * Fraction(float(yv[t, k])))
                exact = sum(terms, Fraction(0))
                mag = float(sum(abs(x) for x in terms))
                err = abs(float(Fraction(float(out[t, j, k])) - exact))
                bound = 1.01 * (n + 1) * U32 * mag
                if dt == "bf16":
                    bound += 2.0 ** -8 * abs(float(exact)) * 1.01
                assert err <= bound, (t, j, k, err, bound)


def test_write_mix_orientation_row_stochastic_preserves_stream_sum():
    """With y = 0, sum_j H'_j = sum_i H_i (sum_j A[i,j]): a matrix whose ROWS sum
    to 1 preserves the per-token stream sum; one whose columns sum to 1 does
    not. This fixes which index of A is the source stream."""
    T, n, d = 32, 4, 64
    H = gen.normal(91, (T, n, d))
    y = np.zeros((T, d), np.float32)
    P = np.abs(gen.normal(92, (T, n, n))) + 0.1
    rows = (P / P.sum(-1, keepdims=True)).astype(np.float32)
    cols = (P / P.sum(-2, keepdims=True)).astype(np.float32)
    b = np.ones((T, n), np.float32)
    s_in = H.astype(np.float64).sum(1)
    scale = np.abs(H.astype(np.float64)).sum(1)
    s_rows = oracle.write_mix(H, y, rows, b, "f32").astype(np.float64).sum(1)
    s_cols = oracle.write_mix(H, y, cols, b, "f32").astype(np.float64).sum(1)
    assert np.max(np.abs(s_rows - s_in) / scale) < 2e-6
    assert np.max(np.abs(s_cols - s_in) / scale) > 1e-2


def test_doubly_stochastic_mix_preserves_stream_sum():
    """The property the mHC constraint exists for: with a (converged) doubly
    stochastic A and y = 0, the per-token sum over streams is unchanged."""
    T, n, d = 64, 4, 128
    H = gen.normal(95, (T, n, d))
    A = oracle.sinkhorn(gen.normal(96, (T, n, n)).astype(np.float64), 500, f64=True)
    A = A.astype(np.float32)
    out = oracle.write_mix(H, np.zeros((T, d), np.float32), A, np.ones((T, n), np.float32), "f32")
    s_in = H.astype(np.float64).sum(1)
    scale = np.abs(H.astype(np.float64)).sum(1)
    assert np.max(np.abs(out.astype(np.float64).sum(1) - s_in) / scale) < 2e-6


def test_write_mix_in_place_equals_out_of_place():
    T, n, d = 8, 4, 32
    H = gen.to_storage(gen.normal(97, (T, n, d)), "bf16")
    y = gen.to_storage(gen.normal(98, (T, d)), "bf16")
    a, A, b = gen.static_params(97, n)
    ref = oracle.write_mix(H, y, A, b, "bf16")
    Hc = H.copy()
    oracle.write_mix(Hc, y, A, b, "bf16", out=Hc)
    assert np.array_equal(Hc, ref)


# --------------------------------------------------------------------------
# read mix + pre-norm RMSNorm
# --------------------------------------------------------------------------

def _exact_rmsnorm(h, g, eps):
    """x_k = h_k / sqrt(mean(h^2) + eps) * g_k with exact sums and 50-digit sqrt."""
    getcontext().prec = 50
    hf = [Fraction(float(v)) for v in h]
    ss = sum((v * v for v in hf), Fraction(0))
    mean = ss / len(hf) + Fraction(float(np.float32(eps)))
    den = (Decimal(mean.numerator) / Decimal(mean.denominator)).sqrt()
    return [float(Decimal(v.numerator) / Decimal(v.denominator) / den) * float(gk)
            for v, gk in zip(hf, g)]


@pytest.mark.parametrize("n", [1, 2, 4])
@pytest.mark.parametrize("dt", ["f32", "bf16"])
def test_read_rmsnorm_brute_force(n, dt):
    T, d = 3, 16
    H = gen.to_storage(gen.normal(101 + n, (T, n, d)), dt)
    a = gen.normal(102 + n, (T, n))
    g = gen.uniform(103, (d,), 0.5, 1.5)
    x = f32_of(oracle.read_rmsnorm(H, a, g, 1e-6, dt), dt)
    Hv = f32_of(H, dt)
    for t in range(T):
        h = [sum((Fraction(float(a[t, i])) * Fraction(float(Hv[t, i, k])) for i in range(n)),
                 Fraction(0)) for k in range(d)]
        want = _exact_rmsnorm([float(v) for v in h], g, 1e-6)
        rms = math.sqrt(sum(w * w for w in want) / d)
        for k in range(d):
            tol = 2e-5 * (abs(want[k]) + rms)
            if dt == "bf16":
                tol += 2.0 ** -8 * abs(want[k])
            assert abs(x[t, k] - want[k]) <= tol, (t, k, x[t, k], want[k])


def test_read_rmsnorm_matches_torch_rms_norm():
    """Read with a = e_0 is RMSNorm of stream 0: compare with the library's
    rms_norm in fp64."""
    T, n, d = 16, 4, 256
    H = gen.normal(111, (T, n, d))
    g = gen.uniform(112, (d,), 0.5, 1.5)
    a = np.array([1.0, 0.0, 0.0, 0.0], np.float32)
    x = oracle.read_rmsnorm(H, a, g, 1e-6, "f32").astype(np.float64)
    ref = torch.nn.functional.rms_norm(torch.from_numpy(H[:, 0].astype(np.float64)), (d,),
                                       weight=torch.from_numpy(g.astype(np.float64)),
                                       eps=float(np.float32(1e-6))).numpy()
    assert np.max(np.abs(x - ref) / (np.abs(ref) + 1e-3)) < 1e-6


def test_rmsnorm_closed_forms():
    """Constant vector c: x = c / sqrt(c^2 + eps) * g. A large eps separates
    eps-inside-the-root from the other placements; the 1/d of the mean is
    separated by d > 1."""
    d = 64
    for c, eps in ((0.5, 0.25), (3.0, 1e-6), (-2.0, 4.0)):
        H = np.full((1, 1, d), c, np.float32)
        g = gen.uniform(121, (d,), 0.5, 1.5)
        x = oracle.read_rmsnorm(H, np.ones(1, np.float32), g, eps, "f32").astype(np.float64)
        want = c / math.sqrt(c * c + float(np.float32(eps))) * g.astype(np.float64)
        assert np.max(np.abs(x[0] - want) / np.abs(want)) < 4 * U32
    # scale invariance: with eps = 0, doubling h leaves x bit-identical
    H = gen.normal(122, (4, 1, d))
    one = np.ones(1, np.float32)
    x1 = oracle.read_rmsnorm(H, one, None, 0.0, "f32")
    x2 = oracle.read_rmsnorm(H * np.float32(2), one, None, 0.0, "f32")
    assert np.array_equal(x1, x2)
    # rms of x / g is 1 (up to eps)
    g = gen.uniform(123, (d,), 0.5, 1.5)
    x = oracle.read_rmsnorm(H, one, g, 1e-6, "f32").astype(np.float64)
    r = np.sqrt(np.mean((x / g) ** 2, axis=-1))
    assert np.max(np.abs(r - 1.0)) < 1e-5


# --------------------------------------------------------------------------
# the whole step: identity initialisation and n = 1
# --------------------------------------------------------------------------

@pytest.mark.parametrize("dt", ["f32", "bf16"])
def test_identity_init_reproduces_single_stream_bitwise(dt):
    """With the n streams copies of one and a = e_0, A = I, b = 1, an HC stack
    computes exactly the one-stream pre-norm residual stack x + f(RMSNorm(x))
    (f = tanh here), and all n streams stay equal. Three layers deep."""
    T, n, d = 64, 4, 1024
    H = gen.copied_streams(1, T, n, d, dt)
    a, A, b = gen.identity_params(n)
    gains = [gen.gain(1, d, layer) for layer in range(4)]
    eps = 1e-6
    x = oracle.read_rmsnorm(H, a, gains[0], eps, dt)
    single = H[:, 0].copy()
    for layer in range(3):
        y = oracle.block_tanh(x, dt)
        H, x = oracle.write_then_read(H, y, A, b, a, gains[layer + 1], eps, dt)
        single = oracle.single_stream_layer(single, gains[layer], eps, dt)
        for j in range(n):
            assert np.array_equal(H[:, j], single), (layer, j)


def test_n1_is_textbook_prenorm_residual():
    """n = 1 with a = A = b = 1 is x + tanh(RMSNorm(x) g): check it against the
    library's rms_norm and tanh in fp64 (fp32 storage; one step)."""
    T, d = 32, 512
    x0 = gen.normal(131, (T, 1, d))
    g = gen.uniform(132, (d,), 0.5, 1.5)
    one = np.ones(1, np.float32)
    xn = oracle.read_rmsnorm(x0, one, g, 1e-6, "f32")
    y = oracle.block_tanh(xn, "f32")
    H1 = oracle.write_mix(x0, y, np.ones((1, 1), np.float32), one, "f32")
    t0 = torch.from_numpy(x0[:, 0].astype(np.float64))
    ref = t0 + torch.tanh(torch.nn.functional.rms_norm(
        t0, (d,), weight=torch.from_numpy(g.astype(np.float64)), eps=float(np.float32(1e-6))))
    assert np.max(np.abs(H1[:, 0] - ref.numpy())) < 1e-5


def test_fused_step_equals_write_then_read_composition():
    T, n, d = 16, 4, 256
    H = gen.to_storage(gen.normal(141, (T, n, d)), "bf16")
    y = gen.to_storage(gen.normal(142, (T, d)), "bf16")
    L = gen.normal(143, (T, n, n)); rl = gen.normal(144, (T, n))
    b = np.ones(n, np.float32)
    g = gen.uniform(145, (d,), 0.5, 1.5)
    H2, x2 = oracle.write_then_read(H, y, L, b, rl, g, 1e-6, "bf16", K=20,
                                    mix_logits=True, read_logits=True)
    A = oracle.sinkhorn(L, 20)
    a = oracle.softmax(rl)
    H1 = oracle.write_mix(H, y, A, b, "bf16")
    x1 = oracle.read_rmsnorm(H1, a, g, 1e-6, "bf16")
    assert np.array_equal(H1, H2) and np.array_equal(x1, x2)


# --------------------------------------------------------------------------
# the pages' own worked arithmetic
# --------------------------------------------------------------------------

def test_state_size_worked_example():
    """16 KB / 64 KB per token per boundary at d = 8192 bf16, 48 KB more, ~4 MB
    at 64 tokens in flight ("What four streams cost per token")."""
    with open(os.path.join(HERE, "golden", "state_sizes.json")) as f:
        g = json.load(f)
    from hyper_connections_stream_b200 import traffic
    one = traffic.state_bytes_per_token(1, g["d"], g["bytes_per_element"])
    four = traffic.state_bytes_per_token(g["n"], g["d"], g["bytes_per_element"])
    assert one == g["one_stream_bytes_per_token"]
    assert four == g["n_stream_bytes_per_token"]
    assert four - one == g["extra_bytes_per_token"]
    assert four * g["tokens_in_flight"] == g["live_state_bytes"]


# --------------------------------------------------------------------------
# input-dependent mixing logits
# --------------------------------------------------------------------------

@pytest.mark.parametrize("dt", ["f32", "bf16"])
def test_mix_logits_against_library_matmul(dt):
    """z = rms-normalised flattened streams times W^T, checked against the
    library's fp64 matmul and norm."""
    T, n, d = 9, 4, 96
    P = n * n + 2 * n
    H = gen.to_storage(gen.normal(151, (T, n, d)), dt)
    W = gen.to_storage(gen.normal(152, (P, n * d), std=0.05), dt)
    z = oracle.mix_logits(H, W, 1e-6, dt)
    u = torch.from_numpy(f32_of(H, dt).reshape(T, n * d))
    Wt = torch.from_numpy(f32_of(W, dt))
    ref = torch.nn.functional.rms_norm(u, (n * d,), eps=float(np.float32(1e-6))) @ Wt.T
    assert np.max(np.abs(z - ref.numpy())) < 1e-12 * (1 + np.max(np.abs(ref.numpy())))


def test_mix_logits_closed_forms():
    """A one-hot weight row picks a single stream value times r; a constant
    token gives z = c / sqrt(c^2 + eps) * sum of the row."""
    T, n, d = 3, 2, 16
    K = n * d
    H = gen.normal(153, (T, n, d))
    W = np.zeros((3, K), np.float32)
    W[0, 5] = 1.0          # stream 0, channel 5
    W[1, d + 2] = -2.0     # stream 1, channel 2
    W[2, :] = 0.5
    z = oracle.mix_logits(H, W, 0.0, "f32")
    u = H.reshape(T, K).astype(np.float64)
    r = 1.0 / np.sqrt(np.mean(u * u, axis=1))
    assert np.allclose(z[:, 0], r * u[:, 5], rtol=1e-14)
    assert np.allclose(z[:, 1], -2.0 * r * u[:, d + 2], rtol=1e-14)
    c = np.full((1, n, d), 0.75, np.float32)
    zc = oracle.mix_logits(c, W, 0.25, "f32")
    want = 0.75 / math.sqrt(0.75 ** 2 + 0.25) * np.array([0.0, 0.0, 0.5 * K])
    want[0] = 0.75 / math.sqrt(0.75 ** 2 + 0.25)
    want[1] = -2.0 * 0.75 / math.sqrt(0.75 ** 2 + 0.25)
    assert np.allclose(zc[0], want, rtol=1e-14)


# --------------------------------------------------------------------------
# stack ends: expansion into n copies, collapse by a weighted sum
# ("Tencent open-sources Hy4 Preview at 770B -- Identity Hyper-Connections",
# TL;DR and residual-design table: the streams start as copies of one)
# --------------------------------------------------------------------------

@pytest.mark.parametrize("dt", ["f32", "bf16"])
def test_expand_is_n_copies(dt):
    T, n, d = 5, 3, 24
    x = gen.to_storage(gen.normal(601, (T, d)), dt)
    H = oracle.expand(x, n, dt)
    want = torch.from_numpy(x.view(np.int16) if dt == "bf16" else x).unsqueeze(1).expand(T, n, d)
    got = torch.from_numpy(H.view(np.int16) if dt == "bf16" else H)
    assert torch.equal(got, want)


@pytest.mark.parametrize("n", [1, 2, 4])
@pytest.mark.parametrize("dt", ["f32", "bf16"])
def test_collapse_brute_force_exact_rationals(n, dt):
    T, d = 3, 16
    H = gen.to_storage(gen.normal(611 + n, (T, n, d)), dt)
    w = gen.normal(612 + n, (T, n))
    out = f32_of(oracle.collapse(H, w, dt), dt)
    Hv = f32_of(H, dt)
    for t in range(T):
        for k in range(d):
            terms = [Fraction(float(w[t, i])) * Fraction(float(Hv[t, i, k])) for i in range(n)]
            exact = sum(terms, Fraction(0))
            mag = float(sum(abs(x) for x in terms))
            bound = 1.01 * n * U32 * mag
            if dt == "bf16":
                bound += 2.0 ** -8 * abs(float(exact)) * 1.01
            assert abs(float(Fraction(float(out[t, k])) - exact)) <= bound, (t, k)


def test_collapse_closed_forms():
    """One-hot weights return that stream bit for bit; weights (1, 1) return
    the fp32 sum of the two streams rounded once to bf16 (torch's add and
    round); expand then a one-hot collapse returns the input."""
    T, n, d = 4, 4, 32
    H = gen.to_storage(gen.normal(621, (T, n, d)), "bf16")
    for k in range(n):
        w = np.zeros(n, np.float32)
        w[k] = 1.0
        assert np.array_equal(oracle.collapse(H, w, "bf16"), H[:, k])
    H2 = np.ascontiguousarray(H[:, :2])
    got = oracle.collapse(H2, np.ones(2, np.float32), "bf16")
    tH = torch.from_numpy(H2.view(np.int16)).view(torch.bfloat16).float()
    want = (tH[:, 0] + tH[:, 1]).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(got, want)
    x = gen.to_storage(gen.normal(622, (T, d)), "bf16")
    assert np.array_equal(oracle.collapse(oracle.expand(x, 3, "bf16"),
                                          np.array([0, 1, 0], np.float32), "bf16"), x)


def test_collapse_softmax_logits_against_library_softmax():
    T, n, d = 6, 4, 16
    H = gen.to_storage(gen.normal(631, (T, n, d)), "f32")
    l = gen.normal(632, (T, n))
    got = oracle.collapse(H, l, "f32", read_logits=True).astype(np.float64)
    w = torch.softmax(torch.from_numpy(l.astype(np.float64)), dim=-1).numpy()
    want = np.einsum("ti,tik->tk", w, H.astype(np.float64))
    mag = np.einsum("ti,tik->tk", w, np.abs(H.astype(np.float64)))
    assert np.all(np.abs(got - want) <= 8 * U32 * mag + 1e-30)


def test_expand_then_read_is_prenorm_of_the_input():
    """Copies of x read with weights summing to 1 in dyadic steps (0.25 each)
    mix back to x exactly, so layer 0's block input is RMSNorm(x) g: compare
    with the library's rms_norm in fp64."""
    T, n, d = 8, 4, 128
    x = gen.normal(641, (T, d))
    g = gen.uniform(642, (d,), 0.5, 1.5)
    a = np.full(n, 0.25, np.float32)
    H, xr = oracle.expand_then_read(x, n, a, g, 1e-6, "f32")
    assert np.array_equal(H[:, 3], x)
    ref = torch.nn.functional.rms_norm(torch.from_numpy(x.astype(np.float64)), (d,),
                                       weight=torch.from_numpy(g.astype(np.float64)),
                                       eps=float(np.float32(1e-6))).numpy()
    assert np.max(np.abs(xr - ref) / (np.abs(ref) + 1e-3)) < 1e-6


# --------------------------------------------------------------------------
# the block's output projection (reference for the fused projection + write)
# --------------------------------------------------------------------------

def test_linear_against_library_matmul_and_closed_forms():
    T, k, d = 7, 40, 24
    X = gen.to_storage(gen.normal(801, (T, k)), "bf16")
    W = gen.to_storage(gen.normal(802, (d, k)), "bf16")
    y = oracle.linear(X, W, "bf16")
    ref = torch.from_numpy(f32_of(X, "bf16")) @ torch.from_numpy(f32_of(W, "bf16")).T
    assert np.max(np.abs(y - ref.numpy())) <= 1e-13 * np.max(np.abs(ref.numpy()))
    # identity weights return X; a one-hot row picks one input channel
    I = gen.to_storage(np.eye(k, dtype=np.float32), "bf16")
    assert np.array_equal(oracle.linear(X, I, "bf16"), f32_of(X, "bf16"))
    W1 = np.zeros((2, k), np.float32)
    W1[0, 3] = 1.0
    W1[1, k - 1] = -2.0
    y1 = oracle.linear(X, gen.to_storage(W1, "bf16"), "bf16")
    assert np.array_equal(y1[:, 0], f32_of(X, "bf16")[:, 3])
    assert np.array_equal(y1[:, 1], -2.0 * f32_of(X, "bf16")[:, k - 1])


# --------------------------------------------------------------------------
# backward pass of the fused step, pinned against torch's automatic
# differentiation (fp64) of the forward definition and against invariants
# --------------------------------------------------------------------------

def _torch_step(H, y, A, b, a, g, eps, K, mix_logits, read_logits):
    """The fused step in torch fp64 (no storage rounding), differentiable."""
    if mix_logits:
        M = torch.exp(A)
        for _ in range(K):
            M = M / M.sum(dim=-1, keepdim=True)
            M = M / M.sum(dim=-2, keepdim=True)
        A = M
    if read_logits:
        a = torch.softmax(a, dim=-1)
    Ab = A if A.dim() == 3 else A.expand(H.shape[0], *A.shape)
    bb = b if b.dim() == 2 else b.expand(H.shape[0], *b.shape)
    ab = a if a.dim() == 2 else a.expand(H.shape[0], *a.shape)
    Hp = torch.einsum("tij,tik->tjk", Ab, H) + bb[:, :, None] * y[:, None, :]
    h = torch.einsum("tj,tjk->tk", ab, Hp)
    r = 1.0 / torch.sqrt((h * h).mean(dim=-1, keepdim=True) + eps)
    return Hp, h * r * g


@pytest.mark.parametrize("n,mix,read,per_token", [(4, True, True, True), (4, False, False, False),
                                                  (2, True, False, True), (1, False, True, True),
                                                  (8, True, True, True), (3, False, False, True)])
def test_backward_against_autograd(n, mix, read, per_token):
    T, d, K, eps = 5, 24, 7, 1e-3
    H = gen.normal(1101 + n, (T, n, d))
    y = gen.normal(1102, (T, d))
    shapeA = (T, n, n) if per_token else (n, n)
    shape_v = (T, n) if per_token else (n,)
    A = gen.normal(1103, shapeA, std=0.7 if mix else 0.5)
    b = gen.normal(1104, shape_v, mean=1.0, std=0.1)
    a = gen.normal(1105, shape_v, std=0.7 if read else 0.5)
    g = gen.uniform(1106, (d,), 0.5, 1.5)
    dHo = gen.normal(1107, (T, n, d))
    dx = gen.normal(1108, (T, d))
    got = oracle.write_then_read_backward(H, y, A, b, a, g, eps, "f32", dHo, dx, K=K,
                                          mix_logits=mix, read_logits=read)
    tt = {k: torch.tensor(v.astype(np.float64), requires_grad=True)
          for k, v in dict(H=H, y=y, A=A, b=b, a=a, g=g).items()}
    Hp, x = _torch_step(tt["H"], tt["y"], tt["A"], tt["b"], tt["a"], tt["g"],
                        float(np.float32(eps)), K, mix, read)
    loss = (Hp * torch.from_numpy(dHo.astype(np.float64))).sum() + \
        (x * torch.from_numpy(dx.astype(np.float64))).sum()
    loss.backward()

    def close(mine, ref, what, tol=2e-5):
        ref = ref.detach().numpy()
        scale = np.max(np.abs(ref)) + 1e-30
        assert np.max(np.abs(mine - ref)) <= tol * scale, (what, np.max(np.abs(mine - ref)) / scale)

    close(got["dH"], tt["H"].grad, "dH")
    close(got["dy"], tt["y"].grad, "dy")
    close(got["dg"], tt["g"].grad, "dg")
    # per-token parameter gradients; a shared parameter's gradient is their sum
    for key, name in (("dA", "A"), ("db", "b"), ("da", "a")):
        mine = got[key] if per_token else got[key].sum(axis=0)
        close(mine, tt[name].grad, key)


def test_backward_invariants():
    """A row shift of the Sinkhorn logits leaves the projection unchanged, so
    each row of dL sums to 0; the softmax's shift invariance makes dl sum to 0;
    with eps = 0, g = 1 and no gradient at H', dh is orthogonal to h."""
    T, n, d, K = 6, 4, 32, 20
    H = gen.normal(1111, (T, n, d))
    y = gen.normal(1112, (T, d))
    L = gen.normal(1113, (T, n, n))
    b = gen.normal(1114, (T, n), mean=1.0, std=0.1)
    l = gen.normal(1115, (T, n))
    dx = gen.normal(1116, (T, d))
    out = oracle.write_then_read_backward(H, y, L, b, l, None, 0.0, "f32", None, dx, K=K,
                                          mix_logits=True, read_logits=True)
    assert np.max(np.abs(out["dA"].sum(axis=-1))) < 1e-9 * (1 + np.max(np.abs(out["dA"])))
    assert np.max(np.abs(out["da"].sum(axis=-1))) < 1e-9 * (1 + np.max(np.abs(out["da"])))
    # standalone Sinkhorn backward equals the one inside the step
    dA = gen.normal(1117, (T, n, n)).astype(np.float64)
    dL = oracle.sinkhorn_backward(L, dA, K)
    assert np.max(np.abs(dL.sum(axis=-1))) < 1e-12 * (1 + np.max(np.abs(dL)))
    # dh orthogonal to h: through da (= sum_k dh_k H'_j,k) with a one-hot read,
    # sum_j a_j da_j = sum_k dh_k h_k = 0
    a1 = np.zeros(n, np.float32)
    a1[2] = 1.0
    o2 = oracle.write_then_read_backward(H, y, L, b, a1, None, 0.0, "f32", None, dx, K=K,
                                         mix_logits=True, read_logits=False)
    scale = np.max(np.abs(o2["da"]))
    assert np.max(np.abs(o2["da"][:, 2])) < 1e-6 * scale


def test_backward_finite_differences():
    """Central differences of the oracle's own forward (fp32 storage) in a few
    random directions agree with the analytic backward."""
    T, n, d, K, eps = 3, 2, 16, 5, 1e-3
    H = gen.normal(1121, (T, n, d))
    y = gen.normal(1122, (T, d))
    L = gen.normal(1123, (T, n, n))
    b = gen.normal(1124, (T, n), mean=1.0, std=0.1)
    l = gen.normal(1125, (T, n))
    g = gen.uniform(1126, (d,), 0.5, 1.5)
    dHo = gen.normal(1127, (T, n, d))
    dx = gen.normal(1128, (T, d))
    grads = oracle.write_then_read_backward(H, y, L, b, l, g, eps, "f32", dHo, dx, K=K,
                                            mix_logits=True, read_logits=True)

    def f(H_, y_, L_, l_):
        Hp, x = oracle.write_then_read(H_.astype(np.float32), y_.astype(np.float32), L_, b,
                                       l_, g, eps, "f32", K=K, mix_logits=True, read_logits=True)
        return float(np.sum(Hp.astype(np.float64) * dHo) + np.sum(x.astype(np.float64) * dx))

    rng = np.random.default_rng(3)
    for name, base, grad in (("H", H, grads["dH"]), ("y", y, grads["dy"]), ("L", L, grads["dA"]),
                             ("l", l, grads["da"])):
        v = rng.standard_normal(base.shape)
        hstep = 1e-2
        args = dict(H_=H, y_=y, L_=L, l_=l)
        key = {"H": "H_", "y": "y_", "L": "L_", "l": "l_"}[name]
        plus = dict(args); plus[key] = (base + hstep * v).astype(np.float32)
        minus = dict(args); minus[key] = (base - hstep * v).astype(np.float32)
        fd = (f(**plus) - f(**minus)) / (2 * hstep)
        an = float(np.sum(grad * v))
        assert abs(fd - an) <= 2e-3 * (abs(an) + 1.0), (name, fd, an)


def test_backward_read_logit_gradient_conditioning():
    """Sets the GPU bar for the read-logit gradient under bf16 storage. With
    logit-mode parameters the exp of the Sinkhorn and softmax definitions may
    differ by an ulp between two correct implementations; a small fraction of
    the recomputed H' then rounds to the adjacent bf16 value and the per-token
    sums move. The oracle's own gradients, with its logits moved by 6e-8
    relative, show the size of that: dA and db stay far inside 2e-4 of their
    largest magnitude, da (a difference of near-equal sums in the softmax
    backward) moves by 1e-5 to 1e-3 of its largest magnitude -- above the
    2e-4 bar of the other gradients, under the 1e-3 bar the GPU tests use."""
    T, n, d, dt = 200, 4, 1024, "bf16"
    H = gen.to_storage(gen.normal(1901, (T, n, d)), dt)
    y = gen.to_storage(gen.normal(1902, (T, d)), dt)
    L = gen.normal(1903, (T, n, n))
    b = gen.normal(1904, (T, n), mean=1.0, std=0.1)
    l = gen.normal(1905, (T, n))
    g = gen.uniform(1906, (d,), 0.5, 1.5)
    dHo = values(gen.to_storage(gen.normal(1907, (T, n, d)), dt), dt)
    dx = values(gen.to_storage(gen.normal(1908, (T, d)), dt), dt)
    ref = oracle.write_then_read_backward(H, y, L, b, l, g, 1e-6, dt, dHo, dx, K=20,
                                          mix_logits=True, read_logits=True)
    rng = np.random.default_rng(19)
    L2 = (L + rng.choice([-1, 0, 1], L.shape) * 6e-8).astype(np.float32)
    l2 = (l + rng.choice([-1, 0, 1], l.shape) * 6e-8).astype(np.float32)
    alt = oracle.write_then_read_backward(H, y, L2, b, l2, g, 1e-6, dt, dHo, dx, K=20,
                                          mix_logits=True, read_logits=True)
    spread = {k: float(np.max(np.abs(alt[k] - ref[k])) / np.max(np.abs(ref[k])))
              for k in ("dA", "db", "da")}
    assert spread["dA"] < 2e-5 and spread["db"] < 1e-4, spread
    assert 1e-5 < spread["da"] < 1e-3, spread


# ---- all-reduce of the block output (the fused reduce + write) ----

def test_reduce_partials_is_the_rank_order_sum_rounded_once():
    """Pins reduce_partials to what the reading fixes: a sum (exact on small
    integers), taken left to right in fp32 (2^24 + 1 + 1 keeps 2^24 in that
    order, gives 2^24 + 2 in the other), rounded to bf16 once at the end
    (1 + 2^-8 + 2^-8 is 1 + 2^-7 exactly in fp32; rounding after each add would
    give 1), and one partial passes through unchanged."""
    rng = np.random.default_rng(2024)
    ints = rng.integers(-30, 31, size=(8, 5, 16))
    parts = [oracle.round_to(v.astype(np.float32), "bf16") for v in ints]
    got = oracle.to_f32(oracle.reduce_partials(parts, "bf16"), "bf16")
    assert np.array_equal(got, ints.sum(axis=0).astype(np.float32))

    big = np.float32(2.0 ** 24)
    f = [np.array([big], np.float32), np.array([1.0], np.float32), np.array([1.0], np.float32)]
    assert oracle.reduce_partials(f, "f32")[0] == big
    assert oracle.reduce_partials(f[::-1], "f32")[0] == big + 2

    one, tiny = np.array([1.0], np.float32), np.array([2.0 ** -8], np.float32)
    b3 = [oracle.round_to(v, "bf16") for v in (one, tiny, tiny)]
    assert oracle.to_f32(oracle.reduce_partials(b3, "bf16"), "bf16")[0] == np.float32(1 + 2.0 ** -7)
    assert oracle.to_f32(oracle.reduce_partials(b3[:2], "bf16"), "bf16")[0] == np.float32(1.0)

    y = oracle.round_to(rng.standard_normal((3, 40)).astype(np.float32), "bf16")
    assert np.array_equal(oracle.reduce_partials([y], "bf16"), y)
