"""CUDA path vs the CPU oracle: threshold calibration, the SVD low-rank predictor, the gathered
gate on the predicted set and the sequential ReGLU FFN."""
import functools

import numpy as np
import pytest
import torch

import oracle
from contextual_sparsity_ffn_b200 import synth
from contextual_sparsity_ffn_b200 import binding as cs
from contextual_sparsity_ffn_b200 import _abi

from gpu_helpers import assert_index_list, dev, dev_layer, run_gate, run_sparse

pytestmark = pytest.mark.gpu


# ------------------------------------------------------------------------------ order statistics

@pytest.mark.parametrize("n,ks", [(1, [1]), (1000, [1, 500, 1000]), (5_636_096, [2_818_048, 3_945_268, 5_072_487])])
def test_kth_smallest_bit_exact(n, ks):
    rng = np.random.default_rng(n)
    v = (np.abs(rng.standard_normal(n)) * 0.3).astype(np.float32)
    v[: min(n, 50)] = v[0]  # ties
    vs = np.sort(v)
    vals = torch.from_numpy(v).cuda()
    out = torch.zeros(1, device="cuda")
    for k in ks:
        cs.kth_smallest(vals, k, out)
        got = out.cpu().numpy()[0]
        assert got.view(np.uint32) == vs[k - 1].view(np.uint32)


def test_kth_smallest_signed_values():
    v = np.array([3.5, -1.0, 0.0, -0.0, 2.0, -7.25, 1e-30, -1e-30], np.float32)
    vals = torch.from_numpy(v).cuda()
    out = torch.zeros(1, device="cuda")
    for k in range(1, len(v) + 1):
        cs.kth_smallest(vals, k, out)
        assert out.item() == np.sort(v)[k - 1]


def test_kth_on_oracle_activations_bit_exact():
    spec, _, xc = synth.tiny_swiglu()
    vals = np.abs(oracle.gate_activation(xc, spec)).ravel().astype(np.float32)
    k = oracle.order_statistic_rank(0.5, vals.size)
    out = torch.zeros(1, device="cuda")
    cs.kth_smallest(torch.from_numpy(vals).cuda(), k, out)
    assert out.cpu().numpy()[0].view(np.uint32) == np.sort(vals)[k - 1].view(np.uint32)


@pytest.mark.parametrize("s", [0.0, 0.5, 0.7, 0.9, 1.0])
def test_calibrate_global_tiny(s):
    spec, _, xc = synth.tiny_swiglu()
    layer = dev_layer(spec)
    t_out = torch.zeros(1, device="cuda")
    cs.calibrate_threshold(layer, dev(xc), s, _abi.CAL_GLOBAL_ABS_ACT, t_out)
    t_ref = oracle.calibrate_global(xc, spec, s)
    assert t_out.item() == pytest.approx(t_ref, rel=1e-5, abs=1e-7)


@pytest.mark.parametrize("s", [0.5, 0.7, 0.9])
def test_calibrate_global_7b(s):
    spec, _, xc = synth.llama2_7b_swiglu(0, n_eval=1, n_calib=512)
    layer = dev_layer(spec)
    t_out = torch.zeros(1, device="cuda")
    cs.calibrate_threshold(layer, dev(xc), s, _abi.CAL_GLOBAL_ABS_ACT, t_out)
    a = np.abs(oracle.gate_activation(xc, spec))
    t_ref = oracle.calibrate_global(xc, spec, s)
    assert t_out.item() == pytest.approx(t_ref, rel=1e-5)
    # the GPU's t hits the requested sparsity on the calibration set
    frac = float((a <= t_out.item()).mean())
    assert abs(frac - s) < 1e-4


# ------------------------------------------------------------------------------ SVD predictor

@functools.lru_cache(maxsize=None)
def reglu_case(d, h, r, n_calib, q=0.9):
    """Workload-2 style layer with oracle SVD factors rounded to bf16 (inputs to both sides)."""
    spec, x, xc = synth.reglu_sparse(0, d=d, h=h, n_eval=4, n_calib=n_calib)
    urt, vr = oracle.svd_factors(spec.w_gate, r)
    urt_b = synth.bf16_bits(urt.astype(np.float32))
    vr_b = synth.bf16_bits(vr.astype(np.float32))
    tau = oracle.calibrate_per_neuron(xc, urt_b, vr_b, spec.bias, q)
    return spec, x, xc, urt_b, vr_b, tau


def _pred_band(p, tau, rms):
    return (np.abs(p - tau[None, :]) < 1e-3 * np.maximum(np.abs(tau), rms)[None, :]).any(axis=0)


@pytest.mark.parametrize("d,h,r", [(1024, 2048, 128), (4096, 11008, 256), (4096, 11008, 1024)])
def test_per_neuron_calibration(d, h, r):
    spec, x, xc, urt, vr, tau_ref = reglu_case(d, h, r, 512)
    layer = dev_layer(spec)
    tau = torch.zeros(h, device="cuda")
    cs.calibrate_threshold(layer, dev(xc), 0.9, _abi.CAL_PER_NEURON_PRED, tau, u_rt=dev(urt), v_r=dev(vr))
    p = oracle.predict(xc, urt, vr, spec.bias)
    rms = np.sqrt(np.mean(p * p, axis=0))
    np.testing.assert_allclose(tau.cpu().numpy(), tau_ref, rtol=1e-4, atol=1e-5 * rms.max())


@pytest.mark.parametrize("d,h,r,n", [(1024, 2048, 128, 512), (4096, 11008, 256, 512), (1024, 1000, 64, 100)])
@pytest.mark.parametrize("R", [0.0, 0.8, 0.95, 1.0])
def test_per_neuron_recall_calibration(d, h, r, n, R):
    """CSFFN_CAL_PER_NEURON_RECALL against oracle.recall_thresholds on the same calibration
    vectors: tau per neuron (+inf where nothing has to be predicted), wherever the active set is
    unambiguous (no vector with z within rounding of 0); and the recall the GPU's thresholds reach
    on the oracle's p and z.  n = 100 is not a power of two (the sort pads it)."""
    spec, x, xc, urt, vr, _ = reglu_case(d, h, r, n)
    layer = dev_layer(spec)
    tau = torch.zeros(h, device="cuda")
    cs.calibrate_threshold(layer, dev(xc), R, _abi.CAL_PER_NEURON_RECALL, tau, u_rt=dev(urt), v_r=dev(vr))
    got = tau.cpu().numpy().astype(np.float64)
    p = oracle.predict(xc, urt, vr, spec.bias)
    z = oracle.gate_preactivation(xc, spec)
    ref = oracle.recall_thresholds(p, z, R)
    zrms = np.sqrt(np.mean(z * z))
    clear = ~(np.abs(z) < 1e-4 * zrms).any(axis=0)
    assert clear.mean() > 0.5
    inf_ref = np.isinf(ref)
    assert np.array_equal(np.isinf(got)[clear], inf_ref[clear])
    if R == 0.0:
        assert np.all(np.isposinf(got))
        return
    fin = clear & ~inf_ref
    assert fin.any()
    prms = np.sqrt(np.mean(p * p, axis=0))
    np.testing.assert_allclose(got[fin], ref[fin], rtol=1e-4, atol=1e-5 * prms.max())
    # the recall reached on the calibration set by every neuron with a clear active set: at least
    # c_i = ceil(R m_i) of its m_i active vectors predicted.  Each threshold sits just below one
    # vector's output, which the fp32 and fp64 sums may put on either side of it, so a vector within
    # rounding of tau counts as predicted.
    act = (z > 0)[:, clear]
    tol = 1e-5 * prms.max()
    hit = (p[:, clear] > got[clear][None, :] - tol) & act
    need = np.array([oracle.order_statistic_rank(R, int(m)) for m in act.sum(axis=0)])
    assert (hit.sum(axis=0) >= need).all()
    assert hit.sum() >= R * act.sum()
    # the thresholds (+inf included) drive the predictor as any others: its candidate list on four
    # other tokens against the oracle's predicted set, outside the rounding band
    ws = cs.new_workspace(layer, 4, r)
    cand_idx = torch.full((h,), -1, dtype=torch.int32, device="cuda")
    cand_count = torch.zeros(1, dtype=torch.int32, device="cuda")
    cs.predict_lowrank(layer, dev(x), dev(urt), dev(vr), tau, cand_idx, cand_count, ws)
    assert cs.check_status(ws) == 0
    P = cand_idx[:int(cand_count.item())].cpu().numpy()
    assert_index_list(P, h)
    pe = oracle.predict(x, urt, vr, spec.bias)
    band = _pred_band(pe, np.where(np.isinf(got), 0.0, got), prms) & ~np.isinf(got)
    pm = np.zeros(h, bool)
    pm[P] = True
    assert np.array_equal(pm[~band], oracle.union_mask(oracle.predicted_mask(pe, got))[~band])


@pytest.mark.parametrize("d,h,r", [(1024, 2048, 128), (4096, 11008, 256), (4096, 11008, 1024)])
@pytest.mark.parametrize("B", [1, 4])
def test_predict_gate_reglu_sequential(d, h, r, B):
    spec, x, xc, urt, vr, tau_ref = reglu_case(d, h, r, 512)
    x = x[:B]
    layer = dev_layer(spec)
    ws = cs.new_workspace(layer, B, r)
    tau = torch.from_numpy(tau_ref.astype(np.float32)).cuda()
    tau64 = tau.cpu().numpy().astype(np.float64)
    cand_idx = torch.full((h,), -1, dtype=torch.int32, device="cuda")
    cand_count = torch.zeros(1, dtype=torch.int32, device="cuda")
    xd = dev(x)
    cs.predict_lowrank(layer, xd, dev(urt), dev(vr), tau, cand_idx, cand_count, ws)
    assert cs.check_status(ws) == 0
    nP = int(cand_count.item())
    P = cand_idx[:nP].cpu().numpy()
    assert_index_list(P, h)
    # predicted set vs oracle, outside the band
    p = oracle.predict(x, urt, vr, spec.bias)
    p_cal = oracle.predict(xc, urt, vr, spec.bias)
    rms = np.sqrt(np.mean(p_cal * p_cal, axis=0))
    pm_ref = oracle.union_mask(oracle.predicted_mask(p, tau64))
    band = _pred_band(p, tau64, rms)
    got = np.zeros(h, bool)
    got[P] = True
    assert np.array_equal(got[~band], pm_ref[~band])
    assert 0.02 < nP / h < (0.5 if B == 1 else 0.9)
    # gathered gate on P (ReLU, t = 0), then up/down on A
    idx, a_val, bufs = run_gate(layer, x, 0.0, ws=ws, cand=(cand_idx, cand_count))
    assert_index_list(idx, h)
    assert set(idx.tolist()) <= set(P.tolist())
    z = oracle.gate_preactivation(x, spec)
    zrms = np.sqrt(np.mean(z * z))
    amask_gpu = np.zeros((B, h), bool)
    amask_gpu[:, idx] = a_val != 0.0
    pred_tok = np.zeros((B, h), bool)
    pred_tok[:, P] = True  # union of predicted rows: every token's gate runs on it
    a_ref = pred_tok & (z > 0)
    clear = np.abs(z) > 1e-3 * zrms
    assert np.array_equal(amask_gpu[clear], a_ref[clear])
    out = run_sparse(layer, bufs)
    ref, _ = oracle.reglu_sequential(x, spec, amask_gpu)
    assert oracle.rel_l2(out, ref) <= 1e-4


def test_predictor_full_rank_is_the_gate():
    """At full rank the predicted set with tau = 0 is {z > 0} (up to bf16 factor rounding)."""
    d, h = 256, 512
    spec = synth.make_layer(57, 0, d, h, "bf16", "relu", bias_mean_std=(-0.3, 0.1))
    x = synth.make_tokens(57, 0, synth.ROLE_EVAL, 1, d, "bf16", rms_normalise=True)
    urt, vr = oracle.svd_factors(spec.w_gate, d)
    urt_b, vr_b = synth.bf16_bits(urt.astype(np.float32)), synth.bf16_bits(vr.astype(np.float32))
    layer = dev_layer(spec)
    ws = cs.new_workspace(layer, 1, d)
    tau = torch.zeros(h, device="cuda")
    ci = torch.zeros(h, dtype=torch.int32, device="cuda")
    cc = torch.zeros(1, dtype=torch.int32, device="cuda")
    cs.predict_lowrank(layer, dev(x), dev(urt_b), dev(vr_b), tau, ci, cc, ws)
    P = ci[: int(cc.item())].cpu().numpy()
    z = oracle.gate_preactivation(x, spec)[0]
    got = np.zeros(h, bool)
    got[P] = True
    clear = np.abs(z) > 0.05 * np.sqrt(np.mean(z * z))
    assert np.array_equal(got[clear], (z > 0)[clear])


@pytest.mark.parametrize("d,h,r", [(1024, 2048, 128), (4096, 11008, 256)])
@pytest.mark.parametrize("B", [1, 4])
def test_predict_then_one_launch_step(d, h, r, B):
    """csffn_predict_lowrank, then csffn_cats_ffn_forward on the predicted set (ReLU, t = 0): the same
    active set as the gathered gate of the two-call path and the oracle's sequential ReGLU output."""
    spec, x, xc, urt, vr, tau_ref = reglu_case(d, h, r, 512)
    x = x[:B]
    layer = dev_layer(spec)
    ws = cs.new_workspace(layer, B, r)
    tau = torch.from_numpy(tau_ref.astype(np.float32)).cuda()
    ci = torch.full((h,), -1, dtype=torch.int32, device="cuda")
    cc = torch.zeros(1, dtype=torch.int32, device="cuda")
    xd = dev(x)
    cs.predict_lowrank(layer, xd, dev(urt), dev(vr), tau, ci, cc, ws)
    idx = torch.full((h,), -1, dtype=torch.int32, device="cuda")
    cnt = torch.zeros(1, dtype=torch.int32, device="cuda")
    av = torch.zeros(B, h, device="cuda")
    out = torch.full((B, d), float("nan"), device="cuda")
    cs.cats_ffn_forward(layer, xd, 0.0, idx, cnt, av, out, ws, cand_idx=ci, cand_count=cc)
    assert cs.check_status(ws) == 0
    n = int(cnt.item())
    idx_f = idx[:n].cpu().numpy()
    av_f = av[:, :n].cpu().numpy().astype(np.float64)
    out_f = out.cpu().numpy().astype(np.float64)
    assert_index_list(idx_f, h)
    P = ci[:int(cc.item())].cpu().numpy()
    assert set(idx_f.tolist()) <= set(P.tolist())
    # the two-call path on the same predicted set
    idx2, a_val2, bufs = run_gate(layer, x, 0.0, ws=ws, cand=(ci, cc))
    z = oracle.gate_preactivation(x, spec)
    zrms = np.sqrt(np.mean(z * z))
    clear = (np.abs(z) > 1e-3 * zrms).all(axis=0)
    g1, g2 = np.zeros(h, bool), np.zeros(h, bool)
    g1[idx_f], g2[idx2] = True, True
    assert np.array_equal(g1[clear], g2[clear])
    amask = np.zeros((B, h), bool)
    amask[:, idx_f] = av_f != 0.0
    ref, _ = oracle.reglu_sequential(x, spec, amask)
    assert oracle.rel_l2(out_f, ref) <= 1e-4


def test_one_launch_step_empty_candidate_list():
    spec, x, xc, urt, vr, tau_ref = reglu_case(1024, 2048, 128, 512)
    layer = dev_layer(spec)
    ws = cs.new_workspace(layer, 1)
    ci = torch.zeros(spec.h, dtype=torch.int32, device="cuda")
    cc = torch.zeros(1, dtype=torch.int32, device="cuda")  # nothing predicted
    idx = torch.zeros(spec.h, dtype=torch.int32, device="cuda")
    cnt = torch.full((1,), 5, dtype=torch.int32, device="cuda")
    av = torch.zeros(1, spec.h, device="cuda")
    out = torch.full((1, spec.d), float("nan"), device="cuda")
    cs.cats_ffn_forward(layer, dev(x[:1]), 0.0, idx, cnt, av, out, ws, cand_idx=ci, cand_count=cc)
    assert cs.check_status(ws) == 0
    assert int(cnt.item()) == 0 and torch.all(out == 0)


@pytest.mark.parametrize("d,h,r,B,parallel", [(1024, 2048, 128, 1, False), (1024, 2048, 128, 4, False),
                                              (4096, 11008, 256, 1, False), (4096, 11008, 1024, 1, False),
                                              (4096, 11008, 256, 3, False), (1024, 2048, 128, 1, True),
                                              (1024, 2048, 128, 4, True), (4096, 11008, 256, 1, True),
                                              (4096, 11008, 1024, 1, True), (4096, 11008, 256, 3, True)])
def test_one_launch_svd_step(d, h, r, B, parallel):
    """csffn_svd_ffn_forward (sequential pipeline: y = x U_r, then predictor, gate on the predicted
    set, up and down on the kept set) and csffn_svd_ffn_forward_parallel
    (W_up read with W_gate on the predicted set) against the predictor + one-launch-on-candidates
    path and the oracle's sequential and parallel ReGLU."""
    spec, x, xc, urt, vr, tau_ref = reglu_case(d, h, r, 512)
    x = x[:B]
    layer = dev_layer(spec)
    ws = cs.new_workspace(layer, B, r)
    tau = torch.from_numpy(tau_ref.astype(np.float32)).cuda()
    xd, urt_d, vr_d = dev(x), dev(urt), dev(vr)
    idx = torch.full((h,), -1, dtype=torch.int32, device="cuda")
    cnt = torch.zeros(1, dtype=torch.int32, device="cuda")
    av = torch.zeros(B, h, device="cuda")
    out = torch.full((B, d), float("nan"), device="cuda")
    cs.svd_ffn_forward(layer, xd, urt_d, vr_d, tau, 0.0, idx, cnt, av, out, ws, parallel=parallel)
    assert cs.check_status(ws) == 0
    n = int(cnt.item())
    idx1 = idx[:n].cpu().numpy()
    av1 = av[:, :n].cpu().numpy().astype(np.float64)
    out1 = out.cpu().numpy().astype(np.float64)
    assert_index_list(idx1, h)
    # reference active set from the oracle, outside the predictor and gate bands
    p = oracle.predict(x, urt, vr, spec.bias)
    p_cal = oracle.predict(xc, urt, vr, spec.bias)
    rms = np.sqrt(np.mean(p_cal * p_cal, axis=0))
    tau64 = tau.cpu().numpy().astype(np.float64)
    pred = oracle.union_mask(oracle.predicted_mask(p, tau64))
    z = oracle.gate_preactivation(x, spec)
    zrms = np.sqrt(np.mean(z * z))
    active_ref = pred & (z > 0).any(axis=0)
    clear = ~_pred_band(p, tau64, rms) & (np.abs(z) > 1e-3 * zrms).all(axis=0)
    got = np.zeros(h, bool)
    got[idx1] = True
    assert np.array_equal(got[clear], active_ref[clear])
    amask = np.zeros((B, h), bool)
    amask[:, idx1] = av1 != 0.0
    ref, _ = oracle.reglu_sequential(x, spec, amask)
    assert oracle.rel_l2(out1, ref) <= 1e-4
    if not _pred_band(p, tau64, rms).any():  # the predicted set is then the oracle's exactly
        ref_par, a_par = oracle.reglu_parallel(x, spec, np.broadcast_to(pred, (B, h)))
        assert oracle.rel_l2(out1, ref_par) <= 1e-4  # a gate near zero contributes almost nothing
    # the same step as two calls (predictor, then the one-launch step on its candidates)
    ci = torch.zeros(h, dtype=torch.int32, device="cuda")
    cc = torch.zeros(1, dtype=torch.int32, device="cuda")
    cs.predict_lowrank(layer, xd, urt_d, vr_d, tau, ci, cc, ws)
    idx2 = torch.zeros(h, dtype=torch.int32, device="cuda")
    cnt2 = torch.zeros(1, dtype=torch.int32, device="cuda")
    av2 = torch.zeros(B, h, device="cuda")
    out2 = torch.zeros(B, d, device="cuda")
    cs.cats_ffn_forward(layer, xd, 0.0, idx2, cnt2, av2, out2, ws, cand_idx=ci, cand_count=cc)
    got2 = np.zeros(h, bool)
    got2[idx2[:int(cnt2.item())].cpu().numpy()] = True
    assert np.array_equal(got[clear], got2[clear])


@pytest.mark.parametrize("parallel", [False, True])
def test_svd_step_whitened_factors(parallel):
    """Data-whitened factors from the offline stage (contextual_sparsity_ffn_b200.offline, computed on
    the device from the calibration tokens) through csffn_calibrate_threshold (per-neuron tau) and the
    SVD step, against the oracle's predictor on the same bf16 factors and its sequential ReGLU."""
    from contextual_sparsity_ffn_b200 import offline
    d, h, r, B = 4096, 11008, 256, 1
    # More calibration vectors than d: with fewer the whitened factors fit the calibration span and
    # predict almost nothing on other tokens (512 vectors: 0.04% of the neurons on the eval tokens)
    spec, x, xc = synth.reglu_sparse(0, d=d, h=h, n_eval=4, n_calib=8192)
    x = x[:B]
    layer = dev_layer(spec)
    urt_d, vr_d = offline.svd_predictor_factors(layer.w_gate, r, dev(xc).float())
    tau = torch.zeros(h, device="cuda")
    cs.calibrate_threshold(layer, dev(xc), 0.9, _abi.CAL_PER_NEURON_PRED, tau, u_rt=urt_d, v_r=vr_d)
    urt, vr = cs.to_numpy_bits(urt_d), cs.to_numpy_bits(vr_d)
    tau64 = tau.cpu().numpy().astype(np.float64)
    ws = cs.new_workspace(layer, B, r)
    idx = torch.full((h,), -1, dtype=torch.int32, device="cuda")
    cnt = torch.zeros(1, dtype=torch.int32, device="cuda")
    av = torch.zeros(B, h, device="cuda")
    out = torch.full((B, d), float("nan"), device="cuda")
    cs.svd_ffn_forward(layer, dev(x), urt_d, vr_d, tau, 0.0, idx, cnt, av, out, ws, parallel=parallel)
    assert cs.check_status(ws) == 0
    n = int(cnt.item())
    idx1 = idx[:n].cpu().numpy()
    av1 = av[:, :n].cpu().numpy().astype(np.float64)
    assert_index_list(idx1, h)
    p = oracle.predict(x, urt, vr, spec.bias)
    p_cal = oracle.predict(xc[:512], urt, vr, spec.bias)
    rms = np.sqrt(np.mean(p_cal * p_cal, axis=0))
    pred = oracle.union_mask(oracle.predicted_mask(p, tau64))
    z = oracle.gate_preactivation(x, spec)
    clear = ~_pred_band(p, tau64, rms) & (np.abs(z) > 1e-3 * np.sqrt(np.mean(z * z))).all(axis=0)
    got = np.zeros(h, bool)
    got[idx1] = True
    assert np.array_equal(got[clear], (pred & (z > 0).any(axis=0))[clear])
    amask = np.zeros((B, h), bool)
    amask[:, idx1] = av1 != 0.0
    ref, _ = oracle.reglu_sequential(x, spec, amask)
    assert oracle.rel_l2(out.cpu().numpy().astype(np.float64), ref) <= 1e-4
    assert 0.01 < pred.mean() < 0.3  # a predicted set of some hundreds of neurons (about 3.6% here)
