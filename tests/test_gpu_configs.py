"""CUDA path vs the CPU oracle on the two composed workloads: the 32-layer LLaMA-3-8B-shaped FFN
stack (batches 1, 4 and 16, per-layer thresholds calibrated on 512 vectors carried through the
dense stack) and the LLaMA-3-70B-shaped Sirius round (16 one-token sparse drafts at 50% and 90%,
then the dense verify of the chunk), with the round's effective density and the drafts' agreement.

Every layer of every step is checked on the GPU's own input and mask (the per-token masks bit for
bit outside the band ||a| - t| < 1e-3 t, the kept activations, the layer's output); the residual
stream is carried on the GPU and compared at the end with an oracle chain that follows the GPU's
masks.  Host work is done one layer at a time (the weights are regenerated from their seeds) so the
host holds at most one layer in float64.
"""
import dataclasses

import numpy as np
import pytest
import torch

import oracle
from contextual_sparsity_ffn_b200 import _abi
from contextual_sparsity_ffn_b200 import binding as cs
from contextual_sparsity_ffn_b200 import stack
from contextual_sparsity_ffn_b200 import synth

from gpu_helpers import check_values, dev, dev_layer, token_masks

pytestmark = pytest.mark.gpu

N_LAYERS = 32
N_CALIB = 512
STACK_BATCHES = (1, 4, 16)
TOL_LAYER = 1e-4   # one layer's fp32 output on the GPU's own input and mask (bf16 weights)
# The end of the 32-layer residual stream against an independent oracle chain (on the GPU's masks):
# each layer re-rounds RMSNorm(h) to bf16 on each side from residuals that differ by fp32 rounding,
# so elements near a bf16 rounding boundary round differently, the next layer's output moves by
# about 2^-9 per flipped element, and the difference compounds layer over layer (measured 5.4e-3 at
# batch 1).  The exact checks are per layer (each on the GPU's own input, and the chain of inputs
# followed bit for bit); this one only bounds the accumulated drift.
TOL_CHAIN = 2e-2


def f64_layer(spec):
    """The layer with its weights decoded to float64 once (every oracle call then reuses them)."""
    return dataclasses.replace(spec, w_gate=oracle.decode(spec.w_gate), w_up=oracle.decode(spec.w_up),
                               w_down_t=oracle.decode(spec.w_down_t))


def record_masks(rec, h):
    """(xn, idx, a_val, h before, h after) of one layer of one step -> per-token masks [B, h]."""
    xn, idx, a_val, _, _ = rec
    return token_masks(idx, a_val.astype(np.float64), h)


def check_layer_record(rec, ref, t):
    """One layer of one sparse stack step against the oracle on the GPU's own input xn; xn itself
    against the oracle's bf16(RMSNorm(h)) of the GPU's residual (at most one bf16 unit apart, and
    equal almost everywhere)."""
    xn, idx, a_val, before, after = rec
    xn_ref = oracle.round_to_bf16(oracle.rmsnorm(before.astype(np.float64)))
    got = oracle.decode(xn)
    assert np.all(np.abs(got - xn_ref) <= np.abs(xn_ref) * 2.0 ** -7 + 1e-30)
    assert np.mean(got == xn_ref) > 0.99
    assert np.all(np.diff(idx) > 0)
    a_ref = oracle.gate_activation(xn, ref)
    m = token_masks(idx, a_val.astype(np.float64), ref.h)
    check_values(a_val.astype(np.float64), idx, a_ref, m, t)
    delta = after.astype(np.float64) - before.astype(np.float64)
    err = oracle.rel_l2(delta, oracle.sparse_ffn(xn, ref, m))
    assert err <= TOL_LAYER, f"layer output rel L2 {err:.3e}"
    return m


# ------------------------------------------------------------------------------ 32-layer 8B stack

def test_llama3_8b_stack_32_layers():
    """Workload: 32 SwiGLU layers d=4096 h=14336 (LLaMA-3-8B FFN shape), CATS at 50% per layer.

    1. GPU calibration: 512 calibration vectors carried through the dense stack; each layer's t
       from its own RMSNorm'd calibration inputs (csffn_calibrate_threshold, exact order statistic).
    2. One decode step of the sparse stack at B = 1, 4 (one-launch step) and 16 (gate mask, then the
       gathered up/down), the residual accumulated in place.
    3. Host pass, one layer at a time: t of the first and last layer against the oracle on the
       GPU's calibration inputs, two calibration vectors carried through the oracle's dense stack
       against the GPU's last-layer calibration input, every step's layer against the oracle, and
       the final residual against the oracle chain on the GPU's masks.
    """
    layers = [dev_layer(synth.llama3_8b_stack_layer(li)) for li in range(N_LAYERS)]
    h_cal_np = synth.llama3_8b_stack_tokens(N_CALIB, synth.ROLE_CALIB)
    h_cal = torch.from_numpy(h_cal_np).cuda()
    ws16 = cs.new_workspace(layers[0], 16)
    kept = {0: None, N_LAYERS - 1: None}
    ts = stack.calibrate_stack(layers, h_cal, 0.5, ws16, keep_inputs=kept)
    assert cs.check_status(ws16) == 0
    assert all(t > 0 for t in ts)

    h0 = synth.llama3_8b_stack_tokens(max(STACK_BATCHES))
    records, finals = {}, {}
    for B in STACK_BATCHES:
        h = torch.from_numpy(h0[:B].copy()).cuda()
        sb = stack.stack_buffers(layers[0], B)
        rec = []
        stack.sparse_stack(layers, ts, h, sb, record=rec)
        assert cs.check_status(sb.buf.ws) == 0
        records[B], finals[B] = rec, h.double().cpu().numpy()
    del layers
    torch.cuda.empty_cache()

    for B in STACK_BATCHES:  # each layer's residual is the previous layer's output, bit for bit
        rec = records[B]
        assert np.array_equal(rec[0][3], h0[:B])
        for li in range(1, N_LAYERS):
            assert np.array_equal(rec[li][3], rec[li - 1][4])
        assert np.array_equal(finals[B], rec[-1][4].astype(np.float64))

    h_ref = {B: h0[:B].astype(np.float64) for B in STACK_BATCHES}
    cal_ref = h_cal_np[:2].astype(np.float64)
    density = {B: [] for B in STACK_BATCHES}
    for li in range(N_LAYERS):
        ref = f64_layer(synth.llama3_8b_stack_layer(li))
        if li in kept:
            t_ref = oracle.calibrate_global(kept[li], ref, 0.5)
            assert ts[li] == pytest.approx(t_ref, rel=1e-5), f"layer {li}"
        if li == N_LAYERS - 1:  # the calibration inputs really went through the dense stack
            xn_ref = oracle.round_to_bf16(oracle.rmsnorm(cal_ref))
            assert oracle.rel_l2(oracle.decode(kept[li][:2]), xn_ref) <= 1e-2
        cal_ref, _, _ = oracle.stack_layer(cal_ref, ref)
        for B in STACK_BATCHES:
            m = check_layer_record(records[B][li], ref, ts[li])
            density[B].append(oracle.union_mask(m).mean())
            h_ref[B], _, _ = oracle.stack_layer(h_ref[B], ref, mask=m)
        del ref
    for B in STACK_BATCHES:
        err = oracle.rel_l2(finals[B], h_ref[B])
        assert err <= TOL_CHAIN, f"B={B}: end of stack rel L2 {err:.3e}"
    # Thresholds calibrated for 50% keep about half of a token's neurons; a union over 4 or 16
    # tokens keeps more.
    assert 0.35 < np.mean(density[1]) < 0.65
    assert np.mean(density[4]) > np.mean(density[1])
    assert np.mean(density[16]) > np.mean(density[4])


# ------------------------------------------------------------------------------ 70B Sirius round

SIRIUS_T = 16  # tokens per round (the chunk the dense verify takes at once)


@pytest.fixture(scope="module")
def sirius70b():
    """The 70B-shaped layer (d=8192 h=28672) on the device, its 16 round tokens, and the GPU's
    thresholds at 50% and 90% from 512 calibration vectors, each checked against the oracle."""
    spec, x, xc = synth.llama3_70b_swiglu(n_eval=SIRIUS_T, n_calib=N_CALIB)
    layer = dev_layer(spec)
    ref = f64_layer(spec)
    del spec
    ts = {}
    t_dev = torch.zeros(1, device="cuda")
    for s in (0.5, 0.9):
        cs.calibrate_threshold(layer, dev(xc), s, _abi.CAL_GLOBAL_ABS_ACT, t_dev)
        ts[s] = float(t_dev.item())
        assert ts[s] == pytest.approx(oracle.calibrate_global(xc, ref, s), rel=1e-5)
    return layer, ref, x, ts


def run_round(layer, x_np, t):
    """One Sirius round through stack.sirius_round; returns (sparse [T, d], dense [T, d], masks [T, h],
    per-draft (idx, a_val))."""
    T = x_np.shape[0]
    x = dev(x_np)
    buf = cs.DecodeBuffers.new(layer, 1)
    ws_dense = cs.new_workspace(layer, T)
    sparse = torch.full((T, layer.d), float("nan"), device="cuda")
    dense = torch.full((T, layer.d), float("nan"), device="cuda")
    rec = []
    stack.sirius_round(layer, x, t, sparse, dense, buf, ws_dense, record=rec)
    assert cs.check_status(buf.ws) == 0 and cs.check_status(ws_dense) == 0
    masks = np.concatenate([token_masks(idx, a_val.astype(np.float64), layer.h) for idx, a_val in rec])
    return sparse.double().cpu().numpy(), dense.double().cpu().numpy(), masks, rec


@pytest.mark.parametrize("s", [0.5, 0.9])
def test_llama3_70b_sirius_round(sirius70b, s):
    """16 batch-1 sparse drafts (the one-launch step) then the dense verify of the chunk, against
    oracle.sirius_round: the draft masks outside the band, each draft's kept activations, the
    drafts' outputs on the GPU's masks and the verify's output."""
    layer, ref, x, ts = sirius70b
    t = ts[s]
    sparse, dense, masks, rec = run_round(layer, x, t)
    sp_ref, de_ref, m_ref = oracle.sirius_round(x, ref, t)
    a_ref = oracle.gate_activation(x, ref)
    for k, (idx, a_val) in enumerate(rec):
        check_values(a_val.astype(np.float64), idx, a_ref[k:k + 1], masks[k:k + 1], t)
    band = np.abs(np.abs(a_ref) - t) < 1e-3 * t
    assert np.array_equal(masks[~band], m_ref[~band])
    assert oracle.rel_l2(sparse, oracle.sparse_ffn(x, ref, masks)) <= TOL_LAYER
    assert oracle.rel_l2(dense, de_ref) <= TOL_LAYER
    if np.array_equal(masks, m_ref):
        assert oracle.rel_l2(sparse, sp_ref) <= TOL_LAYER
    # each draft keeps about 1 - s of the neurons
    assert abs(masks.mean() - (1.0 - s)) < 0.1


@pytest.mark.parametrize("s", [0.5, 0.9])
def test_llama3_70b_round_statistics(sirius70b, s):
    """The round's effective density and the drafts' agreement with the verify, from the GPU's
    outputs, against the oracle's: the masks may differ only at band positions, each of which moves
    a draft's n_t by one (two of the round's 3 h T rows); the agreement is compared with the
    oracle's on the GPU's masks, and with oracle.sirius_round's own where the masks are equal."""
    layer, ref, x, ts = sirius70b
    t = ts[s]
    sparse, dense, masks, _ = run_round(layer, x, t)
    sp_ref, de_ref, m_ref = oracle.sirius_round(x, ref, t)
    band = np.abs(np.abs(oracle.gate_activation(x, ref)) - t) < 1e-3 * t
    diff = masks != m_ref
    assert not (diff & ~band).any()
    h, n_diff = ref.h, int(diff.sum())
    got, want = oracle.round_effective_density(masks), oracle.round_effective_density(m_ref)
    assert abs(got["effective_density"] - want["effective_density"]) <= 2.0 * n_diff / (3.0 * h * SIRIUS_T) + 1e-12
    assert abs(got["neuron_density"] - want["neuron_density"]) <= n_diff / (h * SIRIUS_T) + 1e-12
    assert abs(got["neuron_density"] - (1.0 - s)) < 0.1

    proj = np.random.default_rng(404).standard_normal((ref.d, 64))
    sp_on_gpu_masks = oracle.sparse_ffn(x, ref, masks)
    ag = oracle.draft_agreement(sparse, dense, proj)
    ag_ref = oracle.draft_agreement(sp_on_gpu_masks, de_ref, proj)
    # outputs within 1e-4 relative move ||s - d|| / ||d|| by about 2e-4 / (its value)
    np.testing.assert_allclose(ag["rel_l2"], ag_ref["rel_l2"], rtol=5e-3)
    # top-1 may differ only where the oracle's top two logits (draft or verify) nearly tie
    def near_tie(y):
        lg = np.sort(y @ proj, axis=1)
        return (lg[:, -1] - lg[:, -2]) <= 1e-3 * np.abs(lg).max(axis=1)
    close = near_tie(sp_on_gpu_masks) | near_tie(de_ref)
    assert np.array_equal(ag["top1"][~close], ag_ref["top1"][~close])
    if n_diff == 0:
        own = oracle.draft_agreement(sp_ref, de_ref, proj)
        np.testing.assert_allclose(ag["rel_l2"], own["rel_l2"], rtol=5e-3)
        assert np.array_equal(ag["top1"][~close], own["top1"][~close])
