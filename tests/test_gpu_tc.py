"""CUDA path vs the CPU oracle: the tensor-core (tcgen05) FFN of up to 16 tokens, dense and masked.

csffn_dense_ffn_forward runs it for bf16 layers with d a multiple of 64 and h a multiple of 8, any
batch 1..16; csffn_cats_ffn_forward runs its masked mode (CATS threshold on the activations, the
union compacted into idx / a_val / count) for the batches past the streaming step's tiers.  The
shapes span one and many 128-neuron tiles, a ragged last tile, a single 64-wide k-block, tiles split
between CTAs, and the 70B verify shape.  Outputs in fp32 are held to 1e-4 relative L2 (the bf16
weights and tokens are exact; v is carried as a bf16 high and low part, about 16 bits).
"""
import numpy as np
import pytest
import torch

import oracle
from contextual_sparsity_ffn_b200 import _abi
from contextual_sparsity_ffn_b200 import binding as cs
from contextual_sparsity_ffn_b200 import synth

from gpu_helpers import assert_index_list, check_values, dev, dev_layer, token_masks

pytestmark = pytest.mark.gpu

TOL = 1e-4


def run_dense(layer, x_np, out_dtype=torch.float32, out_mode=None, out=None, ws=None):
    x = dev(x_np)
    B = x.shape[0]
    ws = ws if ws is not None else cs.new_workspace(layer, B)
    if out is None:
        out = torch.full((B, layer.d), float("nan"), dtype=out_dtype, device="cuda")
    cs.dense_ffn_forward(layer, x, out, ws, out_mode=out_mode)
    assert cs.check_status(ws) == 0
    return out.float().cpu().numpy().astype(np.float64)


def run_cats(layer, x_np, t, ws=None, out_mode=None, out=None):
    x = dev(x_np)
    B = x.shape[0]
    ws = ws if ws is not None else cs.new_workspace(layer, B)
    idx = torch.full((layer.h,), -1, dtype=torch.int32, device="cuda")
    count = torch.full((1,), -7, dtype=torch.int32, device="cuda")
    a_val = torch.zeros(B, layer.h, dtype=torch.float32, device="cuda")
    if out is None:
        out = torch.full((B, layer.d), float("nan"), device="cuda")
    cs.cats_ffn_forward(layer, x, t, idx, count, a_val, out, ws, out_mode=out_mode)
    assert cs.check_status(ws) == 0
    n = int(count.item())
    return (idx[:n].cpu().numpy(), a_val[:, :n].cpu().numpy().astype(np.float64),
            out.float().cpu().numpy().astype(np.float64))


@pytest.mark.parametrize("d,h,B,act", [(64, 16, 1, "silu"), (64, 136, 3, "silu"), (128, 1000, 16, "silu"),
                                       (1024, 2000, 16, "silu"), (640, 1000, 9, "silu"), (2048, 3000, 15, "silu"),
                                       (4096, 1024, 12, "relu"), (4096, 11008, 1, "silu"), (4096, 11008, 2, "silu"),
                                       (4096, 14336, 4, "silu"), (4096, 14336, 16, "silu"), (8192, 2048, 7, "silu")])
def test_tc_dense_matches_oracle(d, h, B, act):
    bias = (-0.5, 0.3) if act == "relu" else None
    spec = synth.make_layer(70, d, d, h, "bf16", act, bias_mean_std=bias)
    x = synth.make_tokens(70, d, synth.ROLE_EVAL, B, d, "bf16", rms_normalise=True)
    out = run_dense(dev_layer(spec), x)
    err = oracle.rel_l2(out, oracle.dense_ffn(x, spec))
    assert err <= TOL, f"rel L2 {err:.3e}"


def test_tc_dense_70b_verify_chunk():
    spec, x, _ = synth.llama3_70b_swiglu(n_eval=16, n_calib=1)
    out = run_dense(dev_layer(spec), x)
    assert oracle.rel_l2(out, oracle.dense_ffn(x, spec)) <= TOL


def test_tc_dense_out_modes_and_repeat():
    """bf16 output, accumulate into a seeded residual, and many calls on one workspace (the split
    tiles' counters return to zero after every call): identical results bit for bit."""
    spec = synth.make_layer(71, 0, 2048, 5632, "bf16")
    x = synth.make_tokens(71, 0, synth.ROLE_EVAL, 6, 2048, "bf16", rms_normalise=True)
    layer = dev_layer(spec)
    ws = cs.new_workspace(layer, 16)
    ref = oracle.dense_ffn(x, spec)
    first = run_dense(layer, x, ws=ws)
    assert oracle.rel_l2(first, ref) <= TOL
    for _ in range(5):
        assert np.array_equal(run_dense(layer, x, ws=ws), first)
    ob = run_dense(layer, x, out_dtype=torch.bfloat16, ws=ws)
    assert oracle.rel_l2(ob, ref) <= 1e-2
    res0 = np.random.default_rng(5).standard_normal((6, 2048)).astype(np.float32)
    res = torch.from_numpy(res0).cuda()
    got = run_dense(layer, x, out=res, out_mode=_abi.OUT_F32_ACCUMULATE, ws=ws)
    assert oracle.rel_l2(got - res0, ref) <= TOL
    # a different batch on the same workspace, then the first again
    x3 = x[:3]
    assert oracle.rel_l2(run_dense(layer, x3, ws=ws), ref[:3]) <= TOL
    assert np.array_equal(run_dense(layer, x, ws=ws), first)


@pytest.mark.parametrize("d,h,B,s", [(4096, 14336, 16, 0.5), (4096, 14336, 5, 0.5), (4096, 11008, 8, 0.9),
                                     (8192, 4096, 3, 0.7), (1024, 2000, 16, 0.5), (64, 136, 12, 0.3)])
def test_tc_cats_masked_matches_oracle(d, h, B, s):
    """csffn_cats_ffn_forward past the streaming step's batch tiers: the union index list (exact
    outside the band), the per-token kept activations and the output against the oracle on the
    GPU's own masks."""
    spec = synth.make_layer(72, d, d, h, "bf16")
    x = synth.make_tokens(72, d, synth.ROLE_EVAL, B, d, "bf16", rms_normalise=True)
    a_ref = oracle.gate_activation(x, spec)
    t = float(np.quantile(np.abs(a_ref), s))
    idx, a_val, out = run_cats(dev_layer(spec), x, t)
    assert_index_list(idx, spec.h)
    m = token_masks(idx, a_val, spec.h)
    check_values(a_val, idx, a_ref, m, t)
    band = (np.abs(np.abs(a_ref) - t) < 1e-3 * t).any(axis=0)
    got = np.zeros(spec.h, bool)
    got[idx] = True
    assert np.array_equal(got[~band], oracle.union_mask(oracle.cats_mask(a_ref, t))[~band])
    assert oracle.rel_l2(out, oracle.sparse_ffn(x, spec, m)) <= TOL


def test_tc_cats_degenerate_thresholds():
    spec = synth.make_layer(73, 0, 1024, 1000, "bf16")
    x = synth.make_tokens(73, 0, synth.ROLE_EVAL, 9, 1024, "bf16", rms_normalise=True)
    layer = dev_layer(spec)
    idx, a_val, out = run_cats(layer, x, 1e9)  # nothing kept
    assert len(idx) == 0 and np.all(out == 0.0)
    idx, a_val, out = run_cats(layer, x, -1.0)  # everything kept: the dense FFN
    assert np.array_equal(idx, np.arange(spec.h, dtype=np.int32))
    assert oracle.rel_l2(out, oracle.dense_ffn(x, spec)) <= TOL
    np.testing.assert_allclose(a_val, oracle.gate_activation(x, spec), rtol=1e-4, atol=1e-6)


def test_tc_cats_accumulate_and_repeat():
    spec = synth.make_layer(74, 0, 4096, 14336, "bf16")
    x = synth.make_tokens(74, 0, synth.ROLE_EVAL, 16, 4096, "bf16", rms_normalise=True)
    a_ref = oracle.gate_activation(x, spec)
    t = float(np.quantile(np.abs(a_ref), 0.5))
    layer = dev_layer(spec)
    ws = cs.new_workspace(layer, 16)
    idx0, a0, out0 = run_cats(layer, x, t, ws=ws)
    for _ in range(3):
        idx1, a1, out1 = run_cats(layer, x, t, ws=ws)
        assert np.array_equal(idx1, idx0) and np.array_equal(a1, a0) and np.array_equal(out1, out0)
    res0 = np.random.default_rng(6).standard_normal((16, 4096)).astype(np.float32)
    res = torch.from_numpy(res0).cuda()
    _, _, got = run_cats(layer, x, t, ws=ws, out=res, out_mode=_abi.OUT_F32_ACCUMULATE)
    assert oracle.rel_l2(got - res0, out0) <= 1e-5
