"""Pins of the CPU oracle to things other than itself (CPU only).

Each pin is chosen so that a plausible slip in the oracle (a dropped term, a
wrong sign, a transposed operand, an off-by-one in the order statistic, >=
for >) fails at least one of them; ``test_planted_mistakes`` plants such
slips into the oracle and checks exactly that.
"""
import json
import math
import os
from fractions import Fraction

import numpy as np
import pytest
import scipy.special
import torch

import oracle
from contextual_sparsity_ffn_b200 import synth

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


# ----------------------------------------------------------------------------- helpers

def _closed(expr: str) -> float:
    return float(eval(expr, {"__builtins__": {}}, {"exp": math.exp}))


def _f64(a):
    return oracle.decode(a)


def _tiny_layer(d, h, dtype="bf16", act="silu", bias=None, seed=100):
    return synth.make_layer(seed, 0, d, h, dtype, act, bias_mean_std=bias)


def _tiny_tokens(n, d, dtype="bf16", seed=100, role=synth.ROLE_EVAL):
    return synth.make_tokens(seed, 0, role, n, d, dtype, rms_normalise=True)


# Brute force: the definition written element by element with Python floats.

def bf_dense_ffn(x, layer, mask=None, pred=None):
    """Per-element loops: out[b][c] = sum_i g[b][i] * W_down^T[i][c]."""
    X, Wg, Wu, Wd = (_f64(v).tolist() for v in (x, layer.w_gate, layer.w_up, layer.w_down_t))
    beta = _f64(layer.bias).tolist() if layer.bias is not None else [0.0] * layer.h
    if not isinstance(X[0], list):
        X = [X]
    out = []
    for b, xb in enumerate(X):
        g = []
        for i in range(layer.h):
            z = beta[i]
            u = 0.0
            for k in range(layer.d):
                z += xb[k] * Wg[i][k]
                u += xb[k] * Wu[i][k]
            if layer.act == "silu":
                a = z * (1.0 / (1.0 + math.exp(-z))) if z > -700 else 0.0
            else:
                a = z if z > 0 else 0.0
            keep = True
            if mask is not None:
                keep = bool(mask[b][i]) if np.ndim(mask) == 2 else bool(mask[i])
            if pred is not None:
                keep = keep and bool(pred[b][i]) and z > 0
            g.append(a * u if keep else 0.0)
        row = []
        for c in range(layer.d):
            acc = 0.0
            for i in range(layer.h):
                acc += g[i] * Wd[i][c]
            row.append(acc)
        out.append(row)
    return np.array(out)


def bf_activations(x, layer):
    X, Wg = _f64(x), _f64(layer.w_gate)
    beta = _f64(layer.bias) if layer.bias is not None else np.zeros(layer.h)
    X = np.atleast_2d(X)
    a = np.zeros((X.shape[0], layer.h))
    for b in range(X.shape[0]):
        for i in range(layer.h):
            z = float(beta[i]) + sum(float(X[b, k]) * float(Wg[i, k]) for k in range(layer.d))
            a[b, i] = z / (1.0 + math.exp(-z)) if layer.act == "silu" else max(z, 0.0)
    return a


# ----------------------------------------------------------------------------- closed form

def _golden_layer(g):
    return synth.LayerSpec(d=g["d"], h=g["h"], dtype="f32", act="silu",
                           w_gate=np.array(g["w_gate"], np.float32),
                           w_up=np.array(g["w_up"], np.float32),
                           w_down_t=np.array(g["w_down_t"], np.float32))


def test_closed_form_swiglu():
    with open(os.path.join(GOLDEN, "swiglu_closed_form.json")) as f:
        g = json.load(f)
    layer = _golden_layer(g)
    x = np.array(g["x"], np.float32)
    a = oracle.gate_activation(x, layer)[0]
    np.testing.assert_allclose(a, [_closed(e) for e in g["activation"]], rtol=1e-14, atol=1e-15)
    np.testing.assert_allclose(oracle.dense_ffn(x, layer)[0], [_closed(e) for e in g["dense_out"]],
                               rtol=1e-13, atol=1e-14)
    for case in g["cases"]:
        out, m = oracle.cats_ffn(x, layer, case["t"])
        assert m[0].tolist() == case["mask"]
        np.testing.assert_allclose(out[0], [_closed(e) for e in case["out"]], rtol=1e-13, atol=1e-14)
    for case in g["calibration"]:
        t = oracle.calibrate_global(x, layer, np.float32(case["s"]))
        assert t == pytest.approx(_closed(case["t"]), rel=1e-14, abs=0)


# ----------------------------------------------------------------------------- library routines

def test_silu_matches_scipy_expit():
    z = np.linspace(-60, 60, 2001)
    np.testing.assert_allclose(oracle.silu(z), z * scipy.special.expit(z), rtol=1e-14, atol=1e-300)
    assert oracle.silu(np.array([-1e4]))[0] == 0.0
    assert oracle.silu(np.array([0.0]))[0] == 0.0


def test_decode_bf16_is_exact():
    v = np.array([1.0, -2.5, 3.140625, 65280.0, 2.0 ** -126, 0.0], np.float32)
    np.testing.assert_array_equal(oracle.decode(synth.bf16_bits(v)), v.astype(np.float64))
    bits = np.arange(0, 0x7F80, 7, dtype=np.uint16)  # positive finite bf16 patterns
    ref = torch.from_numpy(bits.view(np.int16)).view(torch.bfloat16).to(torch.float64).numpy()
    np.testing.assert_array_equal(oracle.decode(bits), ref)


def test_round_to_bf16_is_nearest_even():
    rng = np.random.default_rng(5)
    v = rng.standard_normal(4000) * 10.0 ** rng.integers(-5, 5, 4000)
    r = oracle.round_to_bf16(v)
    f = v.astype(np.float32).astype(np.float64)
    # r is a bf16 value: low 16 bits of its float32 pattern are zero
    assert np.all((r.astype(np.float32).view(np.uint32) & 0xFFFF) == 0)
    ulp = np.spacing(np.abs(r).astype(np.float32)).astype(np.float64) * 2 ** 16
    assert np.all(np.abs(f - r) <= ulp / 2 + 1e-300)


def test_rmsnorm_matches_torch():
    v = np.random.default_rng(1).standard_normal((5, 37))
    ref = torch.nn.functional.rms_norm(torch.from_numpy(v), (37,), eps=oracle.RMS_EPS).numpy()
    np.testing.assert_allclose(oracle.rmsnorm(v), ref, rtol=1e-13)


def test_dense_ffn_matches_torch_reference():
    layer = _tiny_layer(48, 72)
    x = _tiny_tokens(3, 48)
    X, Wg, Wu, Wd = (torch.from_numpy(_f64(v)) for v in (x, layer.w_gate, layer.w_up, layer.w_down_t))
    ref = torch.nn.functional.linear(
        torch.nn.functional.silu(torch.nn.functional.linear(X, Wg)) * torch.nn.functional.linear(X, Wu),
        Wd.T).numpy()
    np.testing.assert_allclose(oracle.dense_ffn(x, layer), ref, rtol=1e-12, atol=1e-15)


# ----------------------------------------------------------------------------- brute force

@pytest.mark.parametrize("d,h,dtype", [(12, 20, "bf16"), (16, 9, "f32"), (64, 40, "bf16")])
def test_dense_ffn_brute_force(d, h, dtype):
    layer = _tiny_layer(d, h, dtype)
    x = _tiny_tokens(2, d, dtype)
    np.testing.assert_allclose(oracle.dense_ffn(x, layer), bf_dense_ffn(x, layer), rtol=1e-12, atol=1e-15)


@pytest.mark.parametrize("d,h", [(12, 20), (64, 40)])
def test_cats_sparse_brute_force(d, h):
    layer = _tiny_layer(d, h)
    x = _tiny_tokens(3, d)
    a = bf_activations(x, layer)
    t = float(np.median(np.abs(a)))
    out, m = oracle.cats_ffn(x, layer, t)
    np.testing.assert_array_equal(m, np.abs(a) > t)
    assert 0 < m.sum() < m.size
    np.testing.assert_allclose(out, bf_dense_ffn(x, layer, mask=np.abs(a) > t), rtol=1e-12, atol=1e-15)


def test_sparse_ffn_arbitrary_masks_brute_force():
    """The masked FFN on masks that no threshold produces (a random per-token mask, as the GPU tests
    pass back in from the kernels' own index lists), a one-row mask broadcast over the tokens, and
    the empty and full masks, against the per-element loops."""
    d, h = 12, 20
    layer = _tiny_layer(d, h)
    x = _tiny_tokens(3, d)
    rng = np.random.default_rng(21)
    m = rng.random((3, h)) < 0.4
    np.testing.assert_allclose(oracle.sparse_ffn(x, layer, m), bf_dense_ffn(x, layer, mask=m), rtol=1e-12,
                               atol=1e-15)
    row = rng.random(h) < 0.5
    np.testing.assert_allclose(oracle.sparse_ffn(x, layer, row), bf_dense_ffn(x, layer, mask=row), rtol=1e-12,
                               atol=1e-15)
    assert np.all(oracle.sparse_ffn(x, layer, np.zeros(h, bool)) == 0.0)
    np.testing.assert_allclose(oracle.sparse_ffn(x, layer, np.ones((3, h), bool)), bf_dense_ffn(x, layer),
                               rtol=1e-12, atol=1e-15)


def test_recall_calibration_of_a_layer_brute_force():
    """calibrate_per_neuron_recall on a tiny ReGLU layer with its own factors: the predictor outputs
    and gate pre-activations recomputed by per-element loops, then the recall property on them (at
    least ceil(R m_i) of neuron i's active calibration vectors predicted, and no larger threshold
    predicting as many; +inf where none is needed)."""
    d, h, r, N = 10, 7, 3, 15
    s = synth.reglu_bias_sigma(d)
    layer = _tiny_layer(d, h, act="relu", bias=(-0.5 * s, 0.5 * s))
    xc = _tiny_tokens(N, d, role=synth.ROLE_CALIB)
    urt, vr = oracle.svd_factors(layer.w_gate, r)
    X, Wg, U, V = _f64(xc), _f64(layer.w_gate), np.asarray(urt), np.asarray(vr)
    beta = _f64(layer.bias)
    p = np.zeros((N, h))
    z = np.zeros((N, h))
    for n in range(N):
        y = [sum(float(X[n, j]) * float(U[k, j]) for j in range(d)) for k in range(r)]
        for i in range(h):
            p[n, i] = sum(y[k] * float(V[i, k]) for k in range(r)) + float(beta[i])
            z[n, i] = sum(float(X[n, j]) * float(Wg[i, j]) for j in range(d)) + float(beta[i])
    for R in (0.0, 0.5, 0.9, 1.0):
        tau = oracle.calibrate_per_neuron_recall(xc, urt, vr, layer, R)
        for i in range(h):
            act = [n for n in range(N) if z[n, i] > 0]
            c = _recall_needed(R, len(act))
            if c == 0:
                assert tau[i] == np.inf
                continue
            margin = 1e-9 * (1.0 + abs(tau[i]))  # the loops and the library sum in different orders
            assert sum(p[n, i] > tau[i] - margin for n in act) >= c
            assert sum(p[n, i] > tau[i] + margin for n in act) < c


def test_reglu_sequential_brute_force():
    d, h = 24, 30
    s = synth.reglu_bias_sigma(d)
    layer = _tiny_layer(d, h, act="relu", bias=(-1.5 * s, 0.5 * s))
    x = _tiny_tokens(2, d)
    rng = np.random.default_rng(3)
    pred = rng.random((2, h)) < 0.5
    out, amask = oracle.reglu_sequential(x, layer, pred)
    z_pos = bf_activations(x, layer) > 0
    np.testing.assert_array_equal(amask, pred & z_pos)
    np.testing.assert_allclose(out, bf_dense_ffn(x, layer, pred=pred), rtol=1e-12, atol=1e-15)


def test_reglu_parallel_brute_force():
    """[SVDP] Table 2 caption / Table 3 "Parallel pipeline": gate and up on P, the product ReLU(z) u
    on P into the down projection: per-element loops, and the active set A = P & (z > 0)."""
    d, h = 24, 30
    s = synth.reglu_bias_sigma(d)
    layer = _tiny_layer(d, h, act="relu", bias=(-1.5 * s, 0.5 * s))
    x = _tiny_tokens(3, d)
    pred = np.random.default_rng(4).random((3, h)) < 0.5
    out, amask = oracle.reglu_parallel(x, layer, pred)
    np.testing.assert_array_equal(amask, pred & (bf_activations(x, layer) > 0))
    np.testing.assert_allclose(out, bf_dense_ffn(x, layer, pred=pred), rtol=1e-12, atol=1e-15)
    # one shared predicted set ([h]) is every token's
    out1, _ = oracle.reglu_parallel(x, layer, pred[0])
    np.testing.assert_allclose(out1, bf_dense_ffn(x, layer, pred=np.broadcast_to(pred[0], (3, h))),
                               rtol=1e-12, atol=1e-15)


def test_round_effective_density_by_hand():
    """[SIRIUS] "Key results" / "Approach", FFN weights: (sum_t (h + 2 n_t) + 3 h) / (3 h T)."""
    m = np.array([[1, 0, 0, 0], [1, 1, 1, 0]], bool)  # T = 2, h = 4, n = (1, 3)
    r = oracle.round_effective_density(m)
    assert r["neuron_density"] == 0.5
    assert r["effective_density"] == pytest.approx(28.0 / 24.0, rel=1e-15)  # (6 + 10 + 12) / 24
    T, h = 16, 10
    assert oracle.round_effective_density(np.ones((T, h), bool))["effective_density"] == pytest.approx(1 + 1 / T)
    assert oracle.round_effective_density(np.zeros((T, h), bool))["effective_density"] == pytest.approx(1 / 3 + 1 / T)


def test_draft_agreement_by_hand():
    proj = np.array([[1.0, 0.0, 0.0], [0.0, 1.0, 0.0]])  # d = 2, V = 3
    sp = np.array([[2.0, 1.0], [0.0, 3.0]])
    de = np.array([[2.0, 0.0], [1.0, 0.0]])
    r = oracle.draft_agreement(sp, de, proj)
    assert r["top1"].tolist() == [True, False]  # arg max 0 vs 0; 1 vs 0
    np.testing.assert_allclose(r["rel_l2"], [0.5, math.sqrt(10.0)], rtol=1e-15)


def test_calibration_exhaustive_count():
    d, h, n = 16, 24, 10
    layer = _tiny_layer(d, h)
    xc = _tiny_tokens(n, d, role=synth.ROLE_CALIB)
    a = bf_activations(xc, layer)
    vals = np.abs(a).ravel()
    M = vals.size
    for s in [0.0, 0.1, 0.5, 0.7, 0.9, 0.99, 1.0]:
        t = oracle.calibrate_global(xc, layer, np.float32(s))
        target = Fraction(float(np.float32(s))) * M
        below = sum(1 for v in vals if v <= t)
        if s == 0.0:
            assert t == 0.0 and below == 0
            continue
        # below is the smallest integer >= s*M (no ties among continuous activations)
        assert below >= target > below - 1
        assert sum(1 for v in vals if v < t) == below - 1
        # strict threshold: exactly M - below activations survive on the calibration set
        assert int(oracle.cats_mask(a, t).sum()) == M - below


def test_order_statistic_rank_is_exact():
    # 0.7 is not representable: ceil(0.7 * 10) in floating point would give 8.
    assert oracle.order_statistic_rank(0.7, 10) == 7
    assert oracle.order_statistic_rank(np.float32(0.7), 10) == 7
    assert oracle.order_statistic_rank(np.float32(0.5), 11) == 6
    assert oracle.order_statistic_rank(0.0, 5) == 0
    assert oracle.order_statistic_rank(1.0, 5) == 5


def test_calibration_matches_numpy_inverted_cdf():
    layer, _, xc = synth.tiny_swiglu()
    vals = np.abs(oracle.gate_activation(xc[:64], layer)).ravel()
    for s in [0.25, 0.5, 0.7, 0.9]:
        t = oracle.calibrate_global(xc[:64], layer, s)
        assert t == np.quantile(vals, s, method="inverted_cdf")


def test_per_neuron_calibration_matches_numpy():
    d, h, n, r = 32, 48, 50, 8
    layer = _tiny_layer(d, h)
    xc = _tiny_tokens(n, d, role=synth.ROLE_CALIB)
    urt, vr = oracle.svd_factors(layer.w_gate, r)
    beta = np.linspace(-1, 1, h).astype(np.float32)
    p = oracle.predict(xc, urt, vr, beta)
    for q in [0.5, 0.9]:
        tau = oracle.calibrate_per_neuron(xc, urt, vr, beta, q)
        np.testing.assert_array_equal(tau, np.quantile(p, q, axis=0, method="inverted_cdf"))
        frac = oracle.predicted_mask(p, tau).mean(axis=0)
        assert np.all(frac <= 1 - q + 1e-12)
    assert np.all(np.isneginf(oracle.calibrate_per_neuron(xc, urt, vr, beta, 0.0)))


def test_predicted_mask_brute_force():
    """[SVDP] Fig. 1 and Fig. 2: token b predicts neuron i iff p[b, i] > tau_i (strict), with tau
    per neuron (broadcast over tokens).  A non-square case (B = 3 tokens, h = 5 neurons) with a tie
    p == tau (inactive), a negative tau (a negative p above it is active) and tau = -inf (always
    active, the k = 0 calibration), against a Python loop and a table written out by hand."""
    p = np.array([[0.5, -1.0, 2.0, 0.0, 3.0],
                  [1.0, -2.0, -0.5, -1e300, -9.0],
                  [0.2, 0.2, 0.2, 0.2, 0.2]])
    tau = np.array([0.5, -1.5, 1.0, -np.inf, 0.2])
    loop = [[p[b][i] > tau[i] for i in range(5)] for b in range(3)]
    by_hand = [[False, True, True, True, True],
               [True, False, False, True, False],
               [False, True, False, True, False]]
    got = oracle.predicted_mask(p, tau)
    assert got.shape == (3, 5) and got.dtype == bool
    assert got.tolist() == loop == by_hand
    # one token: the [1, h] row of the same rule
    assert oracle.predicted_mask(p[1:2], tau).tolist() == [by_hand[1]]


def _recall_needed(R: float, m: int) -> int:
    """Brute force: the fewest of m active vectors whose fraction reaches R (R taken at float32)."""
    r = Fraction(float(np.float32(R)))
    return next(c for c in range(m + 1) if m == 0 or Fraction(c, m) >= r) if m else 0


def test_recall_thresholds_brute_force():
    """Per-neuron thresholds for a target recall ([SVDP] Table 3 "+ Bias calibration", Fig. 2),
    checked by their defining properties on a planted case, not by a retyped formula: among the
    active vectors (z > 0, strictly) at least the brute-force count c is predicted (p > tau), no
    larger threshold still predicts c of them, the inactive vectors' outputs do not move tau, and
    tau = +inf when nothing has to be predicted.  Planted: ties among active outputs, z == 0
    (inactive), inactive vectors holding the largest outputs, a neuron never active, negative p."""
    N, h = 9, 6
    rng = np.random.default_rng(11)
    p = np.round(rng.standard_normal((N, h)), 1)  # one decimal: ties occur
    z = rng.standard_normal((N, h))
    z[:, 3] = -np.abs(z[:, 3])           # neuron 3 never active
    z[0, :] = 0.0                        # z == 0 is inactive
    p[0, :] = 50.0                       # ... and holds the largest output
    p[1, 1] = p[2, 1] = p[4, 1] = 0.7    # ties
    z[[1, 2, 4], 1] = 1.0
    z[5, 2] = -1.0
    p[5, 2] = 40.0                       # an inactive vector with a large output
    for R in (0.0, 0.25, 0.5, 0.6, 0.75, 0.99, 1.0):
        tau = oracle.recall_thresholds(p, z, R)
        assert tau.shape == (h,)
        for i in range(h):
            act = [n for n in range(N) if z[n, i] > 0]
            c = _recall_needed(R, len(act))
            if c == 0:
                assert tau[i] == np.inf
                continue
            kept = sum(p[n, i] > tau[i] for n in act)
            assert kept >= c, (R, i, kept, c)
            above = np.nextafter(tau[i], np.inf)
            assert sum(p[n, i] > above for n in act) < c, (R, i)
        # the inactive vectors' outputs do not matter
        q = p.copy()
        q[z <= 0] = rng.standard_normal(int((z <= 0).sum())) * 100.0
        np.testing.assert_array_equal(oracle.recall_thresholds(q, z, R), tau)
    assert oracle.recall_thresholds(p, z, 1.0)[3] == np.inf
    # written out by hand: active outputs 0.1, 0.5, 0.5, 0.9 (and an inactive 5.0)
    pp = np.array([[0.1], [0.5], [0.5], [0.9], [5.0]])
    zz = np.array([[1.0], [2.0], [0.5], [0.1], [-1.0]])
    below = lambda v: np.nextafter(v, -np.inf)
    assert oracle.recall_thresholds(pp, zz, 0.5)[0] == below(0.5)   # c = 2: 0.5, 0.5, 0.9 kept
    assert oracle.recall_thresholds(pp, zz, 0.75)[0] == below(0.5)  # c = 3
    assert oracle.recall_thresholds(pp, zz, 1.0)[0] == below(0.1)   # c = 4: all active kept
    assert oracle.recall_thresholds(pp, zz, 0.25)[0] == below(0.9)  # c = 1


# ----------------------------------------------------------------------------- SVD

def test_svd_full_rank_reconstructs_gate():
    d, h = 40, 56
    layer = _tiny_layer(d, h)
    urt, vr = oracle.svd_factors(layer.w_gate, min(d, h))
    assert urt.shape == (min(d, h), d) and vr.shape == (h, min(d, h))
    np.testing.assert_allclose(vr @ urt, _f64(layer.w_gate), atol=1e-12)
    x = _tiny_tokens(3, d)
    np.testing.assert_allclose(oracle.predict(x, urt, vr), oracle.gate_preactivation(x, layer), atol=1e-12)
    np.testing.assert_allclose(vr.T @ vr, np.eye(min(d, h)), atol=1e-12)


def test_svd_singular_values_and_truncation_error():
    d, h, r = 40, 56, 10
    w = _f64(_tiny_layer(d, h).w_gate)
    urt, vr = oracle.svd_factors(_tiny_layer(d, h).w_gate, r)
    sv = np.sqrt(np.sort(np.linalg.eigvalsh(w.T @ w))[::-1])  # eigenvalues of W_gate^T W_gate (d x d)
    np.testing.assert_allclose(np.linalg.norm(urt, axis=1), sv[:r], rtol=1e-10)
    # Eckart-Young: Frobenius error of the best rank-r approximation
    err = np.linalg.norm(w - vr @ urt)
    assert err == pytest.approx(np.sqrt(np.sum(sv[r:] ** 2)), rel=1e-10)


def _aniso_tokens(n, d, seed=7, spread=5.0):
    """Rows g A with A = diag(spectrum) Q: a fixed input covariance with eigenvalues spread over a
    factor spread^2, so that the data-whitened and the naive factors differ (float32 operands)."""
    rng = np.random.default_rng(seed)
    q, _ = np.linalg.qr(rng.standard_normal((d, d)))
    spec = np.geomspace(1.0, 1.0 / spread, d)
    return (rng.standard_normal((n, d)) @ (spec[:, None] * q)).astype(np.float32)


def test_whitened_svd_is_the_best_rank_r_fit_on_calibration():
    """With no ridge and N >= d, X (U_r V_r^T) is the truncated SVD of X W_gate^T itself (an
    independent route: X = Q R with orthonormal Q, so the X-weighted optimum is the plain
    Eckart-Young optimum of X W_gate^T), and its error beats the naive factors' on X."""
    d, h, n, r = 24, 40, 200, 6
    layer = _tiny_layer(d, h)
    x = _aniso_tokens(n, d)
    xd, w = _f64(x), _f64(layer.w_gate)
    urt, vr = oracle.svd_factors_whitened(layer.w_gate, r, x, ridge=0.0)
    assert urt.shape == (r, d) and vr.shape == (h, r)
    fit = xd @ urt.T @ vr.T
    u, s, vt = np.linalg.svd(xd @ w.T, full_matrices=False)
    best = (u[:, :r] * s[None, :r]) @ vt[:r, :]
    np.testing.assert_allclose(fit, best, atol=1e-10 * np.abs(best).max())
    err_w = np.linalg.norm(xd @ w.T - fit)
    assert err_w == pytest.approx(np.sqrt(np.sum(s[r:] ** 2)), rel=1e-10)
    urt_n, vr_n = oracle.svd_factors(layer.w_gate, r)
    err_n = np.linalg.norm(xd @ w.T - xd @ urt_n.T @ vr_n.T)
    assert err_w < 0.9 * err_n
    # the predictor reads them as it reads the naive factors
    np.testing.assert_allclose(oracle.predict(x[:3], urt, vr), fit[:3], rtol=1e-12)


def test_whitened_svd_full_rank_and_isotropic_data():
    d, h = 20, 32
    layer = _tiny_layer(d, h)
    w = _f64(layer.w_gate)
    x = _aniso_tokens(60, d)
    urt, vr = oracle.svd_factors_whitened(layer.w_gate, d, x)
    np.testing.assert_allclose(vr @ urt, w, atol=1e-10)  # full rank: exact whatever the data
    # X^T X proportional to I (orthonormal columns, scaled): whitening changes nothing
    q, _ = np.linalg.qr(np.random.default_rng(3).standard_normal((80, d)))
    xi = 2.5 * q
    for r in (3, 7):
        urt_w, vr_w = oracle.svd_factors_whitened(layer.w_gate, r, xi)
        urt_n, vr_n = oracle.svd_factors(layer.w_gate, r)
        np.testing.assert_allclose(vr_w @ urt_w, vr_n @ urt_n, atol=1e-9)
    # the ridge only matters where the calibration rows leave C singular (N < d)
    urt_0, vr_0 = oracle.svd_factors_whitened(layer.w_gate, 5, x, ridge=0.0)
    urt_1, vr_1 = oracle.svd_factors_whitened(layer.w_gate, 5, x)
    np.testing.assert_allclose(vr_1 @ urt_1, vr_0 @ urt_0, atol=1e-4 * np.abs(w).max())


# ----------------------------------------------------------------------------- invariants

def test_reglu_t0_equals_dense():
    layer = _tiny_layer(32, 50, act="relu", bias=(-0.2, 0.1))
    x = _tiny_tokens(4, 32)
    out, m = oracle.cats_ffn(x, layer, 0.0)
    np.testing.assert_allclose(out, oracle.dense_ffn(x, layer), rtol=1e-13, atol=1e-15)
    assert m.sum() < m.size  # some neurons really are off


def test_density_one_equals_dense():
    layer = _tiny_layer(32, 50)
    x = _tiny_tokens(4, 32)
    out, m = oracle.cats_ffn(x, layer, -1.0)
    assert m.all()
    np.testing.assert_allclose(out, oracle.dense_ffn(x, layer), rtol=1e-13, atol=1e-15)


def test_batched_equals_per_token_and_union():
    layer = _tiny_layer(32, 50)
    x = _tiny_tokens(4, 32)
    t = 0.1
    out, m = oracle.cats_ffn(x, layer, t)
    for b in range(4):
        ob, mb = oracle.cats_ffn(x[b], layer, t)
        np.testing.assert_allclose(out[b], ob[0], rtol=1e-13, atol=1e-15)
        np.testing.assert_array_equal(m[b], mb[0])
    u = oracle.union_mask(m)
    np.testing.assert_array_equal(u, m.any(axis=0))
    np.testing.assert_array_equal(oracle.active_indices(u), [i for i in range(50) if m[:, i].any()])


def test_sirius_round_composition():
    layer = _tiny_layer(24, 40)
    x = _tiny_tokens(16, 24)
    sp, de, ms = oracle.sirius_round(x, layer, 0.05)
    np.testing.assert_allclose(de, bf_dense_ffn(x, layer), rtol=1e-12, atol=1e-15)
    np.testing.assert_allclose(sp, bf_dense_ffn(x, layer, mask=ms), rtol=1e-12, atol=1e-15)


def test_stack_layer_residual():
    layer = _tiny_layer(24, 40)
    h0 = np.random.default_rng(2).standard_normal((2, 24))
    h1, xn, m = oracle.stack_layer(h0, layer, t=0.05)
    v = h0 / np.sqrt(np.mean(h0 * h0, axis=1, keepdims=True) + 1e-6)
    np.testing.assert_allclose(xn, v, rtol=2 ** -8)
    np.testing.assert_allclose(h1 - h0, bf_dense_ffn(xn, layer, mask=m), rtol=1e-12, atol=1e-15)


def test_rel_l2():
    assert oracle.rel_l2([[3.0, 4.0]], [[3.0, 4.0]]) == 0.0
    assert oracle.rel_l2([[0.0, 0.0]], [[3.0, 4.0]]) == 1.0
    assert oracle.rel_l2([[0.0]], [[0.0]]) == 0.0


# ----------------------------------------------------------------------------- planted mistakes

PIN_TESTS = [
    lambda: test_closed_form_swiglu(),
    lambda: test_dense_ffn_brute_force(12, 20, "bf16"),
    lambda: test_cats_sparse_brute_force(12, 20),
    lambda: test_reglu_sequential_brute_force(),
    lambda: test_calibration_exhaustive_count(),
    lambda: test_calibration_matches_numpy_inverted_cdf(),
    lambda: test_per_neuron_calibration_matches_numpy(),
    lambda: test_svd_full_rank_reconstructs_gate(),
    lambda: test_svd_singular_values_and_truncation_error(),
    lambda: test_whitened_svd_is_the_best_rank_r_fit_on_calibration(),
    lambda: test_whitened_svd_full_rank_and_isotropic_data(),
    lambda: test_silu_matches_scipy_expit(),
    lambda: test_predicted_mask_brute_force(),
    lambda: test_reglu_parallel_brute_force(),
    lambda: test_round_effective_density_by_hand(),
    lambda: test_draft_agreement_by_hand(),
    lambda: test_recall_thresholds_brute_force(),
    lambda: test_sparse_ffn_arbitrary_masks_brute_force(),
    lambda: test_recall_calibration_of_a_layer_brute_force(),
]


def _mut_silu_sign(z):
    with np.errstate(over="ignore"):
        return z / (1.0 + np.exp(z))


def _mut_no_bias(x, layer):
    return oracle.csffn_oracle._tokens(x) @ oracle.decode(layer.w_gate).T


def _mut_down_untransposed(g, layer):
    w = oracle.decode(layer.w_down_t)
    return g @ w[: g.shape[1], :] if w.shape[0] != g.shape[1] else g @ w.T[:, : w.shape[1]]


def _mut_mask_ge(a, t):
    return np.abs(a) >= t


def _mut_rank_floor(s, m):
    return min(max(math.floor(float(s) * m), 0), m)


def _mut_svd_no_sigma(w_gate, r):
    u, s, vt = np.linalg.svd(oracle.decode(w_gate).T, full_matrices=False)
    return u[:, :r].T.copy(), vt[:r, :].T.copy()


def _mut_whiten_untransposed(w_gate, r, x_cal, ridge=oracle.WHITEN_RIDGE):
    xs = oracle.decode(x_cal)
    c = xs.T @ xs
    c = c + (ridge * np.trace(c) / c.shape[0]) * np.eye(c.shape[0])
    low = np.linalg.cholesky(c)
    u, s, vt = np.linalg.svd(low @ oracle.decode(w_gate).T, full_matrices=False)
    return np.linalg.solve(low, u[:, :r] * s[None, :r]).T.copy(), vt[:r, :].T.copy()


def _mut_whiten_not_mapped_back(w_gate, r, x_cal, ridge=oracle.WHITEN_RIDGE):
    xs = oracle.decode(x_cal)
    c = xs.T @ xs
    c = c + (ridge * np.trace(c) / c.shape[0]) * np.eye(c.shape[0])
    low = np.linalg.cholesky(c)
    u, s, vt = np.linalg.svd(low.T @ oracle.decode(w_gate).T, full_matrices=False)
    return (u[:, :r] * s[None, :r]).T.copy(), vt[:r, :].T.copy()


def _mut_pred_ge(p, tau):
    return p >= np.asarray(tau, dtype=np.float64)[None, :]


def _mut_pred_tau_negated(p, tau):
    return p > -np.asarray(tau, dtype=np.float64)[None, :]


def _mut_pred_tau_token_axis(p, tau):
    return p > np.asarray(tau, dtype=np.float64)[:, None]


def _mut_up_uses_gate(x, layer):
    return oracle.csffn_oracle._tokens(x) @ oracle.decode(layer.w_gate).T


def _mut_reglu_ignores_pred(x, layer, pred_mask):
    z = oracle.gate_preactivation(x, layer)
    a_mask = z > 0.0
    out = oracle.down_projection(np.where(a_mask, z, 0.0) * oracle.up_projection(x, layer), layer)
    return out, a_mask


def _mut_parallel_ignores_pred(x, layer, pred_mask):
    z = oracle.gate_preactivation(x, layer)
    g = oracle.relu(z) * oracle.up_projection(x, layer)
    return oracle.down_projection(g, layer), z > 0.0


def _mut_parallel_no_relu(x, layer, pred_mask):
    z = oracle.gate_preactivation(x, layer)
    p = np.broadcast_to(np.asarray(pred_mask, bool), z.shape)
    return oracle.down_projection(np.where(p, z * oracle.up_projection(x, layer), 0.0), layer), p & (z > 0)


def _mut_density_no_verify(masks):
    m = np.asarray(masks, dtype=bool)
    T, h = m.shape
    n = m.sum(axis=1).astype(np.float64)
    return {"neuron_density": float(n.mean() / h), "effective_density": float(np.sum(h + 2.0 * n) / (3.0 * h * T))}


def _mut_agreement_argmin(sparse_out, dense_out, proj):
    s, dn, r = (np.atleast_2d(np.asarray(v, dtype=np.float64)) for v in (sparse_out, dense_out, proj))
    return {"rel_l2": np.linalg.norm(s - dn, axis=1) / np.linalg.norm(dn, axis=1),
            "top1": np.argmin(s @ r, axis=1) == np.argmin(dn @ r, axis=1)}


def _mut_recall_all_vectors(p, z, recall):
    tau = np.full(p.shape[1], np.inf)
    for i in range(p.shape[1]):
        act = np.sort(p[:, i])
        c = oracle.order_statistic_rank(recall, act.size)
        if c > 0:
            tau[i] = np.nextafter(act[act.size - c], -np.inf)
    return tau


def _mut_recall_at_value(p, z, recall):
    tau = np.full(p.shape[1], np.inf)
    for i in range(p.shape[1]):
        act = np.sort(p[z[:, i] > 0, i])
        c = oracle.order_statistic_rank(recall, act.size)
        if c > 0:
            tau[i] = act[act.size - c]
    return tau


def _mut_recall_floor(p, z, recall):
    tau = np.full(p.shape[1], np.inf)
    for i in range(p.shape[1]):
        act = np.sort(p[z[:, i] > 0, i])
        c = math.floor(float(np.float32(recall)) * act.size)
        if c > 0:
            tau[i] = np.nextafter(act[act.size - c], -np.inf)
    return tau


def _mut_recall_zero_active(p, z, recall):
    tau = np.full(p.shape[1], np.inf)
    for i in range(p.shape[1]):
        act = np.sort(p[z[:, i] >= 0, i])
        c = oracle.order_statistic_rank(recall, act.size)
        if c > 0:
            tau[i] = np.nextafter(act[act.size - c], -np.inf)
    return tau


MUTANTS = {
    "silu_sign": ("silu", _mut_silu_sign),
    "dropped_bias": ("gate_preactivation", _mut_no_bias),
    "down_transposed": ("down_projection", _mut_down_untransposed),
    "mask_ge": ("cats_mask", _mut_mask_ge),
    "rank_floor": ("order_statistic_rank", _mut_rank_floor),
    "svd_no_sigma": ("svd_factors", _mut_svd_no_sigma),
    "whiten_untransposed": ("svd_factors_whitened", _mut_whiten_untransposed),
    "whiten_not_mapped_back": ("svd_factors_whitened", _mut_whiten_not_mapped_back),
    "up_uses_gate": ("up_projection", _mut_up_uses_gate),
    "reglu_ignores_pred": ("reglu_sequential", _mut_reglu_ignores_pred),
    "pred_ge": ("predicted_mask", _mut_pred_ge),
    "pred_tau_negated": ("predicted_mask", _mut_pred_tau_negated),
    "pred_tau_token_axis": ("predicted_mask", _mut_pred_tau_token_axis),
    "parallel_ignores_pred": ("reglu_parallel", _mut_parallel_ignores_pred),
    "parallel_no_relu": ("reglu_parallel", _mut_parallel_no_relu),
    "density_no_verify": ("round_effective_density", _mut_density_no_verify),
    "agreement_argmin": ("draft_agreement", _mut_agreement_argmin),
    "recall_all_vectors": ("recall_thresholds", _mut_recall_all_vectors),
    "recall_at_value": ("recall_thresholds", _mut_recall_at_value),
    "recall_floor": ("recall_thresholds", _mut_recall_floor),
    "recall_zero_active": ("recall_thresholds", _mut_recall_zero_active),
}


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_planted_mistakes(name, monkeypatch):
    attr, fn = MUTANTS[name]
    monkeypatch.setattr(oracle.csffn_oracle, attr, fn)
    monkeypatch.setattr(oracle, attr, fn)
    failed = 0
    for pin in PIN_TESTS:
        try:
            pin()
        except Exception:  # an assertion or a shape error both mean the pin caught it
            failed += 1
    assert failed > 0, f"no pin caught the planted mistake {name}"
