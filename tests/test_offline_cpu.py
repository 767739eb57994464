"""The offline SVD predictor factors (contextual_sparsity_ffn_b200.offline) against the oracle (CPU).

"SVD Contextual Sparsity Predictors for Fast LLM Inference", Fig. 1 (offline stage), Table 3
(naive SVD, "+ Data whitening") and Fig. 5 (ROC-AUC of data-aware against naive SVD).  The
factors are compared through U_r V_r^T, which does not depend on the signs of the singular
vectors that the two linear-algebra libraries pick.
"""
import numpy as np
import pytest
import torch

import oracle
from contextual_sparsity_ffn_b200 import offline, synth


def _torch_operand(a: np.ndarray) -> torch.Tensor:
    """The stored operand as a CPU tensor: bf16 bit patterns -> torch.bfloat16, float32 as is."""
    if a.dtype == np.uint16:
        return torch.from_numpy(a.view(np.int16).copy()).view(torch.bfloat16)
    return torch.from_numpy(a.copy())


def _aniso_tokens(n, d, seed, spread=10.0, mix_seed=5):
    """RMS-normalised rows g A, A = diag(spectrum) Q: token covariance eigenvalues spread over a
    factor spread^2 (float32).  The same A for every seed, so calibration and evaluation tokens
    share one distribution."""
    q, _ = np.linalg.qr(np.random.default_rng(mix_seed).standard_normal((d, d)))
    a = np.geomspace(1.0, 1.0 / spread, d)[:, None] * q
    g = np.random.default_rng(seed).standard_normal((n, d)) @ a
    return (g / np.sqrt(np.mean(g * g, axis=1, keepdims=True))).astype(np.float32)


def _product(u_rt, v_r):
    return np.asarray(v_r, dtype=np.float64) @ np.asarray(u_rt, dtype=np.float64)


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
@pytest.mark.parametrize("d,h,r", [(24, 40, 5), (40, 24, 24), (64, 96, 17)])
def test_naive_factors_match_the_oracle(dtype, d, h, r):
    layer = synth.make_layer(31, 0, d, h, dtype, "relu")
    u_rt, v_r = offline.svd_predictor_factors(_torch_operand(layer.w_gate), r, out_dtype=torch.float64)
    assert tuple(u_rt.shape) == (r, d) and tuple(v_r.shape) == (h, r)
    urt_o, vr_o = oracle.svd_factors(layer.w_gate, r)
    ref = _product(urt_o, vr_o)
    np.testing.assert_allclose(_product(u_rt.numpy(), v_r.numpy()), ref, atol=1e-10 * np.abs(ref).max())
    # row norms of U_r^T are the singular values
    np.testing.assert_allclose(u_rt.norm(dim=1).numpy(), np.linalg.norm(urt_o, axis=1), rtol=1e-10)


@pytest.mark.parametrize("n", [16, 200])  # fewer calibration rows than d (the ridge decides), and more
@pytest.mark.parametrize("ridge", [0.0, 1e-6])
def test_whitened_factors_match_the_oracle(n, ridge):
    d, h, r = 32, 48, 6
    if n < d and ridge == 0.0:
        pytest.skip("X^T X is singular without the ridge")
    layer = synth.make_layer(32, 0, d, h, "bf16", "relu")
    x = _aniso_tokens(n, d, seed=1)
    u_rt, v_r = offline.svd_predictor_factors(_torch_operand(layer.w_gate), r, torch.from_numpy(x), ridge=ridge,
                                              out_dtype=torch.float64)
    ref = _product(*oracle.svd_factors_whitened(layer.w_gate, r, x, ridge=ridge))
    np.testing.assert_allclose(_product(u_rt.numpy(), v_r.numpy()), ref, atol=1e-9 * np.abs(ref).max())


def test_factor_dtype_layout_and_errors():
    d, h, r = 32, 40, 8
    layer = synth.make_layer(33, 0, d, h, "bf16", "relu")
    w = _torch_operand(layer.w_gate)
    u_rt, v_r = offline.svd_predictor_factors(w, r)
    assert u_rt.dtype == torch.bfloat16 and v_r.dtype == torch.bfloat16
    assert u_rt.is_contiguous() and v_r.is_contiguous()
    ref = _product(*oracle.svd_factors(layer.w_gate, r))
    got = _product(u_rt.float().numpy(), v_r.float().numpy())
    assert np.linalg.norm(got - ref) <= 1e-2 * np.linalg.norm(ref)  # bf16-rounded factors
    for bad in (0, min(d, h) + 1):
        with pytest.raises(ValueError):
            offline.svd_predictor_factors(w, bad)
    with pytest.raises(ValueError):
        offline.svd_predictor_factors(w, r, torch.zeros(4, d + 1))
    with pytest.raises(ValueError):
        offline.svd_predictor_factors(w[0], r)


def _auroc(score: np.ndarray, label: np.ndarray) -> float:
    """Mean over neurons of P(score of an active case > score of an inactive case) (ties count 1/2)."""
    aucs = []
    for i in range(score.shape[1]):
        pos, neg = score[label[:, i], i], score[~label[:, i], i]
        if len(pos) == 0 or len(neg) == 0:
            continue
        allv = np.concatenate([pos, neg])
        order = np.argsort(allv, kind="mergesort")
        ranks = np.empty(len(allv))
        ranks[order] = np.arange(1, len(allv) + 1)
        # average ranks over ties
        _, inv, cnt = np.unique(allv, return_inverse=True, return_counts=True)
        ranks = (np.bincount(inv, weights=ranks) / cnt)[inv]
        aucs.append((ranks[: len(pos)].sum() - len(pos) * (len(pos) + 1) / 2) / (len(pos) * len(neg)))
    return float(np.mean(aucs))


def test_whitened_predictor_beats_naive_on_anisotropic_tokens(capsys):
    """The predictor quality the data-whitened factors buy (the pages' Fig. 5 comparison): a
    ReGLU layer (tiny shape) whose tokens have a spread-out covariance; factors from 2048
    calibration tokens, per-neuron tau at q = 0.5 on them, scored on 2048 other tokens of the same
    distribution.  Recall of the truly active set at equal predicted density, ROC-AUC of p against
    z > 0, and the relative error of p against z."""
    d, h = 256, 688
    layer = synth.make_layer(34, 0, d, h, "f32", "relu")
    xc, xe = _aniso_tokens(2048, d, seed=1), _aniso_tokens(2048, d, seed=2)
    z = oracle.gate_preactivation(xe, layer)
    active = z > 0
    w = _torch_operand(layer.w_gate)
    rows = []
    for r in (32, 64):
        res = {}
        for name, xcal in (("naive", None), ("whitened", torch.from_numpy(xc))):
            u_rt, v_r = offline.svd_predictor_factors(w, r, xcal, out_dtype=torch.float64)
            u_rt, v_r = u_rt.numpy(), v_r.numpy()
            tau = oracle.calibrate_per_neuron(xc, u_rt, v_r, None, 0.5)
            p = oracle.predict(xe, u_rt, v_r)
            pred = p > tau[None, :]
            res[name] = dict(recall=(pred & active).sum() / active.sum(), density=pred.mean(),
                             auroc=_auroc(p, active), rel_err=np.linalg.norm(p - z) / np.linalg.norm(z))
        rows.append((r, res))
        n, wt = res["naive"], res["whitened"]
        assert abs(wt["density"] - n["density"]) < 0.01
        assert wt["recall"] > n["recall"] + 0.03
        assert wt["auroc"] > n["auroc"] + 0.02
        assert wt["rel_err"] < 0.9 * n["rel_err"]
    with capsys.disabled():
        for r, res in rows:
            print(f"\nr={r}: " + "; ".join(f"{k}: recall {v['recall']:.3f} density {v['density']:.3f} "
                                         f"AUROC {v['auroc']:.3f} rel.err {v['rel_err']:.3f}" for k, v in res.items()))


def test_recall_targeted_thresholds_on_anisotropic_tokens(capsys):
    """Per-neuron thresholds set for a target recall R of the truly active set (the pages' Table 3
    "+ Bias calibration" and Fig. 2, in the reading of oracle.recall_thresholds) on the workload
    above: set on the 2048 calibration tokens, scored on 2048 others.  The recall carries over to
    the held-out tokens, a higher R costs predicted density, and the data-whitened factors reach the
    same recall at a lower density than the naive ones."""
    d, h = 256, 688
    layer = synth.make_layer(34, 0, d, h, "f32", "relu")
    xc, xe = _aniso_tokens(2048, d, seed=1), _aniso_tokens(2048, d, seed=2)
    zc, ze = oracle.gate_preactivation(xc, layer), oracle.gate_preactivation(xe, layer)
    active = ze > 0
    w = _torch_operand(layer.w_gate)
    rows = []
    for r in (32, 64):
        res = {}
        for name, xcal in (("naive", None), ("whitened", torch.from_numpy(xc))):
            u_rt, v_r = offline.svd_predictor_factors(w, r, xcal, out_dtype=torch.float64)
            u_rt, v_r = u_rt.numpy(), v_r.numpy()
            pc, pe = oracle.predict(xc, u_rt, v_r), oracle.predict(xe, u_rt, v_r)
            for R in (0.9, 0.95, 0.99):
                tau = oracle.recall_thresholds(pc, zc, R)
                cal = (pc > tau[None, :]) & (zc > 0)
                assert cal.sum() >= R * (zc > 0).sum()  # reached on the calibration set
                pred = pe > tau[None, :]
                res[(name, R)] = dict(recall=(pred & active).sum() / active.sum(), density=pred.mean())
        rows.append((r, res))
        for R in (0.9, 0.95, 0.99):
            n, wt = res[("naive", R)], res[("whitened", R)]
            assert n["recall"] > R - 0.02 and wt["recall"] > R - 0.02
            assert wt["density"] < n["density"] - 0.01
        for name in ("naive", "whitened"):
            assert res[(name, 0.9)]["density"] < res[(name, 0.95)]["density"] < res[(name, 0.99)]["density"]
    with capsys.disabled():
        for r, res in rows:
            print(f"\nr={r}: " + "; ".join(f"{k[0]} R={k[1]}: recall {v['recall']:.3f} density {v['density']:.3f}"
                                          for k, v in res.items()))


def test_artefacts_round_trip_bit_for_bit(tmp_path):
    layer = synth.make_layer(35, 0, 32, 48, "bf16", "relu")
    u_rt, v_r = offline.svd_predictor_factors(_torch_operand(layer.w_gate), 8)
    tau = torch.linspace(-1.0, 1.0, 48, dtype=torch.float32)
    t = torch.tensor([0.123456789], dtype=torch.float32)
    counts = torch.arange(5, dtype=torch.int32)
    path = str(tmp_path / "layer0.npz")
    offline.save_artefacts(path, u_rt=u_rt, v_r=v_r, tau=tau, t=t, counts=counts)
    got = offline.load_artefacts(path)
    assert set(got) == {"u_rt", "v_r", "tau", "t", "counts"}
    for name, ref in (("u_rt", u_rt), ("v_r", v_r), ("tau", tau), ("t", t), ("counts", counts)):
        assert got[name].dtype == ref.dtype and got[name].shape == ref.shape
        if ref.dtype == torch.bfloat16:
            assert torch.equal(got[name].view(torch.int16), ref.view(torch.int16))
        else:
            assert torch.equal(got[name], ref)
    with pytest.raises(TypeError):
        offline.save_artefacts(path, t=0.5)
