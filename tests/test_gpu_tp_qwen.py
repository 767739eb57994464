"""CUDA path vs the CPU oracle: the tensor-parallel split of a layer (its row blocks run on one GPU
one after another, their fp32 partial outputs summed as the all-reduce would) and the SparseQwen2-7B
FFN shape (d 3584, h 18944, ReGLU): the CATS step at batch 1 and 4, the dense verify, the SVD step
in both pipelines."""
import numpy as np
import pytest
import torch

import oracle
from contextual_sparsity_ffn_b200 import _abi
from contextual_sparsity_ffn_b200 import binding as cs
from contextual_sparsity_ffn_b200 import synth
from contextual_sparsity_ffn_b200 import tensor_parallel as tp

from gpu_helpers import assert_index_list, check_values, dev, dev_layer, token_masks

pytestmark = pytest.mark.gpu

TOL = 1e-4


def run_step(layer, x, t, ws=None):
    B = x.shape[0]
    buf = cs.DecodeBuffers.new(layer, max(B, 1))
    out = torch.full((B, layer.d), float("nan"), device="cuda")
    cs.cats_ffn_forward(layer, x, t, buf.idx, buf.count, buf.a_val, out, buf.ws, out_mode=_abi.OUT_F32)
    assert cs.check_status(buf.ws) == 0
    n = int(buf.count.item())
    return buf.idx[:n].cpu().numpy(), buf.a_val[:B, :n].cpu().numpy().astype(np.float64), out


@pytest.mark.parametrize("world,B", [(2, 1), (4, 1), (2, 4), (3, 2)])
def test_row_blocks_sum_to_the_layer(world, B):
    """Each rank's block of rows through csffn_cats_ffn_forward, the partial outputs summed: the
    layer's output, and the ranks' active lists (moved to layer numbering) the layer's list."""
    spec, _, xc = synth.llama2_7b_swiglu(0, n_eval=1, n_calib=64)
    x_np = synth.make_tokens(82, 0, synth.ROLE_EVAL, B, spec.d, "bf16", rms_normalise=True)
    full = dev_layer(spec)
    x = dev(x_np)
    a_ref = oracle.gate_activation(x_np, spec)
    t = float(np.quantile(np.abs(a_ref), 0.5))
    idx_f, a_f, out_f = run_step(full, x, t)
    total = torch.zeros(B, spec.d, device="cuda")
    idx_parts, a_parts = [], []
    for r in range(world):
        shard = tp.ShardedLayer.from_full(full, world, r)
        buf = cs.DecodeBuffers.new(shard.layer, max(B, 1))
        out = torch.zeros(B, spec.d, device="cuda")
        tp.tp_cats_forward(shard, x, t, out, buf)  # no process group: the partial output alone
        assert cs.check_status(buf.ws) == 0
        n = int(buf.count.item())
        idx_parts.append(tp.global_indices(buf.idx[:n], shard).cpu().numpy())
        a_parts.append(buf.a_val[:B, :n].cpu().numpy().astype(np.float64))
        total += out
    idx = np.concatenate(idx_parts)
    a_val = np.concatenate(a_parts, axis=1)
    assert_index_list(idx.astype(np.int32), spec.h)
    m = token_masks(idx, a_val, spec.h)
    check_values(a_val, idx, a_ref, m, t, atol_rel=1e-5 if B >= 3 else 1e-6)
    band = (np.abs(np.abs(a_ref) - t) < 1e-3 * t).any(axis=0)
    got = np.zeros(spec.h, bool)
    got[idx] = True
    full_set = np.zeros(spec.h, bool)
    full_set[idx_f] = True
    assert np.array_equal(got[~band], full_set[~band])
    assert oracle.rel_l2(total.double().cpu().numpy(), oracle.sparse_ffn(x_np, spec, m)) <= TOL
    if np.array_equal(got, full_set):
        assert oracle.rel_l2(total.double().cpu().numpy(), out_f.double().cpu().numpy()) <= 1e-5


@pytest.mark.parametrize("world", [2, 4])
def test_threshold_from_all_blocks(world):
    """The layer's threshold from the blocks' pooled activations (the values tp_calibrate gathers)
    equals csffn_calibrate_threshold on the whole layer."""
    spec, _, xc = synth.llama2_7b_swiglu(0, n_eval=1, n_calib=64)
    full = dev_layer(spec)
    xcd = dev(xc)
    t_dev = torch.zeros(1, device="cuda")
    cs.calibrate_threshold(full, xcd, 0.7, _abi.CAL_GLOBAL_ABS_ACT, t_dev)
    parts = [tp.local_abs_activations(tp.ShardedLayer.from_full(full, world, r), xcd) for r in range(world)]
    vals = torch.cat(parts, dim=1).reshape(-1).contiguous()
    k = tp._order_statistic_rank(0.7, vals.numel())
    t_out = torch.zeros(1, device="cuda")
    cs.kth_smallest(vals, k, t_out)
    assert t_out.item() == pytest.approx(t_dev.item(), rel=1e-5)
    assert t_out.item() == pytest.approx(oracle.calibrate_global(xc, spec, 0.7), rel=1e-5)


# ------------------------------------------------------------------------------ SparseQwen2 shape

@pytest.fixture(scope="module")
def qwen():
    spec, x, xc = synth.sparse_qwen2_reglu(0, n_eval=16, n_calib=512)
    return spec, x, xc, dev_layer(spec)


@pytest.mark.parametrize("B,s", [(1, 0.5), (1, 0.9), (4, 0.5)])
def test_qwen2_cats_step(qwen, B, s):
    spec, x_all, _, layer = qwen
    x_np = x_all[:B]
    a_ref = oracle.gate_activation(x_np, spec)
    t = float(np.quantile(np.abs(a_ref), s))
    idx, a_val, out = run_step(layer, dev(x_np), t)
    assert_index_list(idx, spec.h)
    m = token_masks(idx, a_val, spec.h)
    check_values(a_val, idx, a_ref, m, t, atol_rel=1e-5 if B >= 3 else 1e-6)  # B >= 3: tensor cores
    assert oracle.rel_l2(out.double().cpu().numpy(), oracle.sparse_ffn(x_np, spec, m)) <= TOL


def test_qwen2_dense_verify(qwen):
    spec, x_all, _, layer = qwen
    out = torch.full((16, spec.d), float("nan"), device="cuda")
    ws = cs.new_workspace(layer, 16)
    cs.dense_ffn_forward(layer, dev(x_all), out, ws)
    assert cs.check_status(ws) == 0
    assert oracle.rel_l2(out.double().cpu().numpy(), oracle.dense_ffn(x_all, spec)) <= TOL


@pytest.mark.parametrize("parallel", [False, True])
def test_qwen2_svd_step(qwen, parallel):
    """Rank-512 predictor (Table 12 of the SVD page lists this FFN shape), per-neuron tau at
    q = 0.9 calibrated on the device, the SVD step against the oracle's sequential ReGLU on the
    GPU's kept set and its predicted set outside the band."""
    spec, x_all, xc, layer = qwen
    x_np = x_all[:1]
    r = 512
    urt, vr = oracle.svd_factors(spec.w_gate, r)
    urt_b, vr_b = synth.bf16_bits(urt.astype(np.float32)), synth.bf16_bits(vr.astype(np.float32))
    urt_d, vr_d = dev(urt_b), dev(vr_b)
    tau = torch.zeros(spec.h, device="cuda")
    cs.calibrate_threshold(layer, dev(xc), 0.9, _abi.CAL_PER_NEURON_PRED, tau, u_rt=urt_d, v_r=vr_d)
    ws = cs.new_workspace(layer, 1, r)
    idx = torch.full((spec.h,), -1, dtype=torch.int32, device="cuda")
    cnt = torch.zeros(1, dtype=torch.int32, device="cuda")
    av = torch.zeros(1, spec.h, device="cuda")
    out = torch.full((1, spec.d), float("nan"), device="cuda")
    cs.svd_ffn_forward(layer, dev(x_np), urt_d, vr_d, tau, 0.0, idx, cnt, av, out, ws, parallel=parallel)
    assert cs.check_status(ws) == 0
    n = int(cnt.item())
    idx1 = idx[:n].cpu().numpy()
    assert_index_list(idx1, spec.h)
    tau64 = tau.cpu().numpy().astype(np.float64)
    p = oracle.predict(x_np, urt_b, vr_b, spec.bias)
    p_cal = oracle.predict(xc[:256], urt_b, vr_b, spec.bias)
    rms = np.sqrt(np.mean(p_cal * p_cal, axis=0))
    pred = oracle.union_mask(oracle.predicted_mask(p, tau64))
    z = oracle.gate_preactivation(x_np, spec)
    band = (np.abs(p - tau64[None, :]) < 1e-3 * np.maximum(np.abs(tau64), rms)[None, :]).any(axis=0)
    clear = ~band & (np.abs(z) > 1e-3 * np.sqrt(np.mean(z * z))).all(axis=0)
    got = np.zeros(spec.h, bool)
    got[idx1] = True
    assert np.array_equal(got[clear], (pred & (z > 0).any(axis=0))[clear])
    amask = np.zeros((1, spec.h), bool)
    amask[:, idx1] = av[:, :n].cpu().numpy() != 0.0
    ref, _ = oracle.reglu_sequential(x_np, spec, amask)
    assert oracle.rel_l2(out.double().cpu().numpy(), ref) <= TOL
    assert 0.02 < pred.mean() < 0.3
