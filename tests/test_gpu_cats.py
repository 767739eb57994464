"""CUDA path vs the CPU oracle: CATS gate mask, gathered sparse FFN, dense FFN, union of masks.

Parity rules: the active-index set is bit-exact outside the band ||a| - t| < 1e-3 t; the output is
then compared with the oracle run on the GPU's own per-token mask.  Max relative L2 error per
output vector: <= 1e-5 for fp32 workloads, <= 1e-2 for bf16 workloads (plus a tighter 1e-4 check
on fp32 outputs of bf16 layers, which any single dropped or wrong neuron would exceed).
"""
import numpy as np
import pytest
import torch

import oracle
from contextual_sparsity_ffn_b200 import synth
from contextual_sparsity_ffn_b200 import binding as cs

from gpu_helpers import (assert_index_list, band_rows, check_values, dev, dev_layer, run_dense, run_gate,
                         run_sparse, token_masks)

pytestmark = pytest.mark.gpu

TOL_F32 = 1e-5
TOL_BF16 = 1e-2
TOL_BF16_F32OUT = 1e-4


def check_cats(spec, x, t, tol, layer=None, out_dtype=torch.float32):
    """Run gate + sparse forward on the GPU and check against the oracle; return (err, density)."""
    layer = layer or dev_layer(spec)
    idx, a_val, bufs = run_gate(layer, x, t)
    assert_index_list(idx, spec.h)
    a_ref = oracle.gate_activation(x, spec)
    m_ref = oracle.cats_mask(a_ref, t)
    union_ref = oracle.union_mask(m_ref)
    band = band_rows(a_ref, t)
    got = np.zeros(spec.h, dtype=bool)
    got[idx] = True
    assert np.array_equal(got[~band], union_ref[~band]), "active set differs outside the band"
    # per-token values: a where the token keeps the neuron, else 0
    m_gpu = token_masks(idx, a_val, spec.h)
    tb = np.abs(np.abs(a_ref) - t) < 1e-3 * abs(t)
    assert np.array_equal(m_gpu[~tb], m_ref[~tb])
    a_sel = np.where(m_gpu, a_ref, 0.0)[:, idx]
    np.testing.assert_allclose(a_val, a_sel, rtol=1e-4, atol=1e-6 * np.abs(a_ref).max())
    out = run_sparse(layer, bufs, out_dtype=out_dtype)
    ref = oracle.sparse_ffn(x, spec, m_gpu)
    err = oracle.rel_l2(out, ref)
    assert err <= tol, f"rel L2 {err:.3e} > {tol}"
    return err, len(idx) / spec.h, out


# ------------------------------------------------------------------------------ tiny fp32 workload

def test_tiny_fp32_each_token():
    spec, x, xc = synth.tiny_swiglu()
    t = oracle.calibrate_global(xc, spec, 0.5)
    layer = dev_layer(spec)
    for b in range(x.shape[0]):
        err, dens, _ = check_cats(spec, x[b:b + 1], t, TOL_F32, layer=layer)
        assert 0.3 < dens < 0.7


def test_tiny_fp32_union_batch16():
    spec, x, xc = synth.tiny_swiglu()
    t = oracle.calibrate_global(xc, spec, 0.5)
    err, dens, out = check_cats(spec, x, t, TOL_F32)
    assert dens > 0.99  # union of 16 independent tokens at 50% is ~1 - 2^-16
    # batched output == each token alone
    layer = dev_layer(spec)
    for b in [0, 7, 15]:
        _, _, ob = check_cats(spec, x[b:b + 1], t, TOL_F32, layer=layer)
        assert oracle.rel_l2(out[b], ob[0]) <= TOL_F32


def test_tiny_fp32_dense():
    spec, x, _ = synth.tiny_swiglu()
    out = run_dense(dev_layer(spec), x)
    assert oracle.rel_l2(out, oracle.dense_ffn(x, spec)) <= TOL_F32


# ------------------------------------------------------------------------------ ragged shapes

@pytest.mark.parametrize("d,h,B", [(520, 1000, 1), (520, 1000, 3), (8, 5, 1), (64, 16, 2), (1032, 33, 5),
                                   (4104, 777, 1)])
def test_ragged_bf16(d, h, B):
    spec = synth.make_layer(50, d, d, h, "bf16")
    x = synth.make_tokens(50, d, synth.ROLE_EVAL, B, d, "bf16", rms_normalise=True)
    a = np.abs(oracle.gate_activation(x, spec))
    t = float(np.quantile(a, 0.5))
    check_cats(spec, x, t, TOL_BF16_F32OUT)
    out = run_dense(dev_layer(spec), x)
    assert oracle.rel_l2(out, oracle.dense_ffn(x, spec)) <= TOL_BF16_F32OUT


@pytest.mark.parametrize("d,h", [(256, 688), (12, 40)])
def test_ragged_fp32(d, h):
    spec = synth.make_layer(51, d, d, h, "f32")
    x = synth.make_tokens(51, d, synth.ROLE_EVAL, 2, d, "f32", rms_normalise=False)
    t = float(np.quantile(np.abs(oracle.gate_activation(x, spec)), 0.7))
    check_cats(spec, x, t, TOL_F32)


# ------------------------------------------------------------------------------ degenerate cases

def test_empty_active_set_gives_zero():
    spec = synth.make_layer(52, 0, 256, 300, "bf16")
    x = synth.make_tokens(52, 0, synth.ROLE_EVAL, 2, 256, "bf16", rms_normalise=True)
    layer = dev_layer(spec)
    idx, a_val, bufs = run_gate(layer, x, 1e9)
    assert len(idx) == 0
    out = run_sparse(layer, bufs)
    assert np.all(out == 0.0)
    # accumulate mode leaves the residual unchanged
    res = torch.arange(2 * 256, dtype=torch.float32, device="cuda").reshape(2, 256)
    keep = res.clone()
    cs.sparse_ffn_forward(layer, bufs["x"], bufs["idx"], bufs["count"], bufs["a_val"], res, bufs["ws"],
                          out_mode=cs._abi.OUT_F32_ACCUMULATE)
    assert torch.equal(res, keep)


def test_all_active_equals_dense():
    spec, x, _ = synth.llama2_7b_swiglu(0, n_eval=2, n_calib=1)
    layer = dev_layer(spec)
    idx, a_val, bufs = run_gate(layer, x, -1.0)
    assert len(idx) == spec.h
    out = run_sparse(layer, bufs)
    assert oracle.rel_l2(out, oracle.dense_ffn(x, spec)) <= TOL_BF16_F32OUT
    assert oracle.rel_l2(out, run_dense(layer, x)) <= TOL_BF16_F32OUT


def test_reglu_t0_equals_dense():
    spec = synth.make_layer(53, 0, 1024, 2000, "bf16", "relu", bias_mean_std=(-0.5, 0.2))
    x = synth.make_tokens(53, 0, synth.ROLE_EVAL, 1, 1024, "bf16", rms_normalise=True)
    layer = dev_layer(spec)
    idx, a_val, bufs = run_gate(layer, x, 0.0)
    z = oracle.gate_preactivation(x, spec)[0]
    clear = np.abs(z) > 1e-4
    got = np.zeros(spec.h, bool)
    got[idx] = True
    assert np.array_equal(got[clear], (z > 0)[clear])
    out = run_sparse(layer, bufs)
    assert oracle.rel_l2(out, oracle.dense_ffn(x, spec)) <= TOL_BF16_F32OUT


def test_batch_zero_writes_zero_count():
    spec = synth.make_layer(54, 0, 64, 40, "bf16")
    layer = dev_layer(spec)
    ws = cs.new_workspace(layer, 1)
    count = torch.full((1,), 5, dtype=torch.int32, device="cuda")
    idx = torch.zeros(40, dtype=torch.int32, device="cuda")
    a_val = torch.zeros(1, 40, device="cuda")
    x = torch.zeros(0, 64, dtype=torch.bfloat16, device="cuda")
    cs._abi.check(cs.load().csffn_gate_mask(layer.ref(), None, 0, 0.1, None, None, cs._ptr(idx), cs._ptr(count),
                                            cs._ptr(a_val), cs._ptr(ws), ws.numel(), cs._stream()), "b0")
    assert int(count.item()) == 0


def test_repeated_calls_reuse_workspace():
    """Epoch-tagged look-back: many launches on one workspace give identical results."""
    spec = synth.make_layer(55, 0, 512, 3000, "bf16")
    x = synth.make_tokens(55, 0, synth.ROLE_EVAL, 1, 512, "bf16", rms_normalise=True)
    layer = dev_layer(spec)
    ws = cs.new_workspace(layer, 4)
    first = None
    for it in range(20):
        t = 0.05 if it % 2 == 0 else 0.2
        idx, a_val, bufs = run_gate(layer, x, t, ws=ws)
        out = run_sparse(layer, bufs)
        if it < 2:
            first = first or {}
            first[t] = (idx.copy(), out.copy())
        else:
            assert np.array_equal(idx, first[t][0])
            assert np.array_equal(out, first[t][1])  # deterministic, bit for bit


def test_bf16_output_mode():
    spec = synth.make_layer(56, 0, 1024, 2048, "bf16")
    x = synth.make_tokens(56, 0, synth.ROLE_EVAL, 2, 1024, "bf16", rms_normalise=True)
    t = float(np.quantile(np.abs(oracle.gate_activation(x, spec)), 0.5))
    check_cats(spec, x, t, TOL_BF16, out_dtype=torch.bfloat16)


# ------------------------------------------------------------------------------ full-size workloads

@pytest.mark.parametrize("s", [0.5, 0.7, 0.9])
def test_llama2_7b_batch1(s):
    spec, x, xc = synth.llama2_7b_swiglu(0, n_eval=2, n_calib=512)
    t = oracle.calibrate_global(xc, spec, s)
    layer = dev_layer(spec)
    for b in range(2):
        err, dens, _ = check_cats(spec, x[b:b + 1], t, TOL_BF16_F32OUT, layer=layer)
        assert abs((1 - dens) - s) < 0.05


def test_llama3_8b_union_batch4_and_16():
    spec = synth.llama3_8b_stack_layer(0)
    x = synth.make_tokens(3, 0, synth.ROLE_EVAL, 16, 4096, "bf16", rms_normalise=True)
    t = float(np.quantile(np.abs(oracle.gate_activation(x, spec)), 0.5))
    layer = dev_layer(spec)
    err4, dens4, out4 = check_cats(spec, x[:4], t, TOL_BF16_F32OUT, layer=layer)
    assert 0.85 < dens4 < 0.99
    err16, dens16, out16 = check_cats(spec, x, t, TOL_BF16_F32OUT, layer=layer)
    assert dens16 > 0.99
    assert oracle.rel_l2(out16[:4], out4) <= TOL_BF16_F32OUT


def test_llama3_70b_batch1_sampled():
    spec, x, _ = synth.llama3_70b_swiglu(n_eval=1, n_calib=1)
    a = np.abs(oracle.gate_activation(x, spec))
    t = float(np.quantile(a, 0.9))
    check_cats(spec, x, t, TOL_BF16_F32OUT)


def test_llama3_70b_dense_verify_chunk():
    # 16 tokens at d = 8192: the tensor-core path (one pass over W_gate / W_up for all tokens)
    spec, x, _ = synth.llama3_70b_swiglu(n_eval=16, n_calib=1)
    out = run_dense(dev_layer(spec), x)
    assert oracle.rel_l2(out, oracle.dense_ffn(x, spec)) <= TOL_BF16_F32OUT


@pytest.mark.parametrize("d,h,B,act", [(1024, 2000, 16, "silu"), (640, 1000, 9, "silu"), (1024, 777, 8, "silu"),
                                       (4096, 1024, 12, "relu"), (128, 16, 16, "silu"), (2048, 3000, 15, "silu")])
def test_dense_token_block_tensor_cores(d, h, B, act):
    """Dense FFN for 8..16 tokens (bf16): tensor-core gate/up and down, ragged neuron tiles,
    partial 512-column chunks, the ReGLU bias; fp32 output to 1e-4, bf16 output to 1e-2."""
    bias = (-0.5, 0.3) if act == "relu" else None
    spec = synth.make_layer(64, d, d, h, "bf16", act, bias_mean_std=bias)
    x = synth.make_tokens(64, d, synth.ROLE_EVAL, B, d, "bf16", rms_normalise=True)
    layer = dev_layer(spec)
    ref = oracle.dense_ffn(x, spec)
    out = run_dense(layer, x)
    assert oracle.rel_l2(out, ref) <= TOL_BF16_F32OUT
    outb = run_dense(layer, x, out_dtype=torch.bfloat16)
    assert oracle.rel_l2(outb, ref) <= TOL_BF16
    # each token's row equals its own batch-1 dense output (CUDA-core GEMV path)
    for b in (0, B - 1):
        one = run_dense(layer, x[b:b + 1])
        assert oracle.rel_l2(out[b:b + 1], one) <= TOL_BF16_F32OUT


# ------------------------------------------------------------------------------ one-launch decode step

def run_fused(layer, x_np, t, out_dtype=torch.float32, ws=None):
    x = dev(x_np if x_np.ndim == 2 else x_np[None, :])
    B = x.shape[0]
    idx = torch.full((layer.h,), -1, dtype=torch.int32, device="cuda")
    count = torch.full((1,), -7, dtype=torch.int32, device="cuda")
    a_val = torch.zeros(B, layer.h, dtype=torch.float32, device="cuda")
    out = torch.full((B, layer.d), float("nan"), dtype=out_dtype, device="cuda")
    ws = ws if ws is not None else cs.new_workspace(layer, B)
    cs.cats_ffn_forward(layer, x, t, idx, count, a_val, out, ws)
    assert cs.check_status(ws) == 0
    n = int(count.item())
    return (idx[:n].cpu().numpy(), a_val[:, :n].cpu().numpy().astype(np.float64),
            out.float().cpu().numpy().astype(np.float64))


@pytest.mark.parametrize("d,h,B,dtype,s", [(256, 688, 1, "f32", 0.5), (520, 1000, 3, "bf16", 0.5),
                                           (4096, 11008, 1, "bf16", 0.5), (4096, 11008, 1, "bf16", 0.9),
                                           (4096, 14336, 4, "bf16", 0.5), (64, 16, 2, "bf16", 0.3),
                                           (8192, 2048, 1, "bf16", 0.7), (1024, 777, 8, "bf16", 0.5),
                                           (1024, 777, 2, "bf16", 0.5), (4096, 11008, 2, "bf16", 0.7)])
def test_fused_decode_matches_oracle_and_two_call_path(d, h, B, dtype, s):
    spec = synth.make_layer(62, d, d, h, dtype)
    x = synth.make_tokens(62, d, synth.ROLE_EVAL, B, d, dtype, rms_normalise=dtype == "bf16")
    a_ref = oracle.gate_activation(x, spec)
    t = float(np.quantile(np.abs(a_ref), s))
    layer = dev_layer(spec)
    idx, a_val, out = run_fused(layer, x, t)
    assert_index_list(idx, h)
    band = band_rows(a_ref, t)
    got = np.zeros(h, bool)
    got[idx] = True
    assert np.array_equal(got[~band], oracle.union_mask(oracle.cats_mask(a_ref, t))[~band])
    m = token_masks(idx, a_val, h)
    check_values(a_val, idx, a_ref, m, t)
    tol = TOL_F32 if dtype == "f32" else TOL_BF16_F32OUT
    assert oracle.rel_l2(out, oracle.sparse_ffn(x, spec, m)) <= tol
    # the two-call path (other kernels, other summation order) gives the same set outside the band,
    # the same values to rounding, and the same output to rounding
    idx2, a_val2, bufs = run_gate(layer, x, t)
    got2 = np.zeros(h, bool)
    got2[idx2] = True
    assert np.array_equal(got[~band], got2[~band])
    if np.array_equal(idx, idx2):
        np.testing.assert_allclose(a_val, a_val2, rtol=1e-5, atol=1e-7 * np.abs(a_ref).max())
    out2 = run_sparse(layer, bufs)
    m2 = token_masks(idx2, a_val2, h)
    assert oracle.rel_l2(out2, oracle.sparse_ffn(x, spec, m2)) <= tol


def test_fused_decode_repeated_and_modes():
    spec, x, xc = synth.llama2_7b_swiglu(0, n_eval=2, n_calib=64)
    t = oracle.calibrate_global(xc, spec, 0.5)
    layer = dev_layer(spec)
    ws = cs.new_workspace(layer, 1)
    first = run_fused(layer, x[:1], t, ws=ws)
    for _ in range(10):  # the ticket and grid counters reset themselves between launches
        again = run_fused(layer, x[:1], t, ws=ws)
        # each row's gate and up are reduced in a fixed order, so the mask and values repeat
        # exactly; rows reach CTAs dynamically, so the output's summation order (and its
        # rounding) may change from launch to launch
        assert np.array_equal(first[0], again[0]) and np.array_equal(first[1], again[1])
        assert oracle.rel_l2(again[2], first[2]) <= 1e-6
    idx, a_val, outb = run_fused(layer, x[:1], t, out_dtype=torch.bfloat16, ws=ws)
    m = token_masks(idx, a_val, spec.h)
    assert oracle.rel_l2(outb, oracle.sparse_ffn(x[:1], spec, m)) <= TOL_BF16
    # accumulate mode adds into the residual
    res = torch.ones(1, spec.d, dtype=torch.float32, device="cuda")
    xd = dev(x[:1])
    bidx = torch.zeros(spec.h, dtype=torch.int32, device="cuda")
    bcnt = torch.zeros(1, dtype=torch.int32, device="cuda")
    bav = torch.zeros(1, spec.h, device="cuda")
    cs.cats_ffn_forward(layer, xd, t, bidx, bcnt, bav, res, ws, out_mode=cs._abi.OUT_F32_ACCUMULATE)
    assert cs.check_status(ws) == 0
    assert oracle.rel_l2(res.double().cpu().numpy() - 1.0, first[2]) <= TOL_BF16_F32OUT


def test_fused_decode_empty_and_all_active():
    spec = synth.make_layer(63, 0, 512, 700, "bf16")
    x = synth.make_tokens(63, 0, synth.ROLE_EVAL, 1, 512, "bf16", rms_normalise=True)
    layer = dev_layer(spec)
    idx, a_val, out = run_fused(layer, x, 1e9)
    assert len(idx) == 0 and np.all(out == 0.0)
    idx, a_val, out = run_fused(layer, x, -1.0)
    assert len(idx) == spec.h
    assert oracle.rel_l2(out, oracle.dense_ffn(x, spec)) <= TOL_BF16_F32OUT


def test_fused_decode_reglu_with_gate_bias():
    spec, x, _ = synth.reglu_sparse(0, d=1024, h=2752, n_eval=3, n_calib=1)
    layer = dev_layer(spec)
    z = oracle.gate_preactivation(x, spec)
    for t in (0.0, float(np.quantile(np.abs(oracle.gate_activation(x, spec)), 0.8))):
        idx, a_val, out = run_fused(layer, x, t)
        assert_index_list(idx, spec.h)
        a_ref = oracle.gate_activation(x, spec)
        band = band_rows(a_ref, t) if t > 0 else np.abs(z).min(axis=0) < 1e-6
        got = np.zeros(spec.h, bool)
        got[idx] = True
        assert np.array_equal(got[~band], oracle.union_mask(oracle.cats_mask(a_ref, t))[~band])
        m = token_masks(idx, a_val, spec.h)
        if t > 0:
            check_values(a_val, idx, a_ref, m, t)
        assert oracle.rel_l2(out, oracle.sparse_ffn(x, spec, m)) <= TOL_BF16_F32OUT


def test_fused_decode_7b_low_threshold_keeps_negative_activations():
    """t = 0.25 < max |SiLU| on the negative side (0.278): neurons with z in about (-2, -0.75)
    are kept too, so the kept set is not one-sided; one-launch and two-call paths against the oracle."""
    spec, x, _ = synth.llama2_7b_swiglu(0, n_eval=1, n_calib=1)
    t = 0.25
    a_ref = oracle.gate_activation(x, spec)
    keep_ref = oracle.union_mask(oracle.cats_mask(a_ref, t))
    assert (a_ref[0][keep_ref] < 0).sum() > 1000  # the case this test is for
    layer = dev_layer(spec)
    band = band_rows(a_ref, t)
    for one_launch in (True, False):
        if one_launch:
            idx, a_val, out = run_fused(layer, x, t)
        else:
            idx, a_val, bufs = run_gate(layer, x, t)
            out = run_sparse(layer, bufs)
        got = np.zeros(spec.h, bool)
        got[idx] = True
        assert np.array_equal(got[~band], keep_ref[~band])
        m = token_masks(idx, a_val, spec.h)
        check_values(a_val, idx, a_ref, m, t)
        assert oracle.rel_l2(out, oracle.sparse_ffn(x, spec, m)) <= TOL_BF16_F32OUT


@pytest.mark.parametrize("pinned", [True, False])
@pytest.mark.parametrize("B", [2, 4])
def test_fused_decode_host_buffers(pinned, B):
    """csffn_cats_ffn_forward_host: tokens in and output out through host memory -- pinned (the step
    reads and writes the mapped host buffers itself) and pageable (staged through the workspace by
    copies) -- checked against the oracle on the call's own mask, and against the device entry
    point's result (bf16 and fp32 outputs).  B = 2 runs the streaming step, B = 4 the tensor-core
    FFN in masked mode."""
    spec, x, xc = synth.llama2_7b_swiglu(0, n_eval=B, n_calib=64)
    t = oracle.calibrate_global(xc, spec, 0.5)
    layer = dev_layer(spec)
    ws = cs.new_workspace(layer, B)
    idx_d, a_val_d, out_d = run_fused(layer, x, t, ws=ws)
    xh = dev(x).cpu()
    if pinned:
        xh = xh.pin_memory()
    for dtype, tol in ((torch.float32, 1e-6), (torch.bfloat16, TOL_BF16)):
        oh = torch.full((B, spec.d), float("nan"), dtype=dtype)
        if pinned:
            oh = oh.pin_memory()
        idx = torch.zeros(spec.h, dtype=torch.int32, device="cuda")
        cnt = torch.zeros(1, dtype=torch.int32, device="cuda")
        av = torch.zeros(B, spec.h, device="cuda")
        cs.cats_ffn_forward_host(layer, xh, t, idx, cnt, av, oh, ws)
        torch.cuda.synchronize()
        assert cs.check_status(ws) == 0
        n = int(cnt.item())
        got_idx = idx[:n].cpu().numpy()
        got_av = av[:, :n].cpu().numpy().astype(np.float64)
        assert_index_list(got_idx, spec.h)
        m = token_masks(got_idx, got_av, spec.h)
        a_ref = oracle.gate_activation(x, spec)
        check_values(got_av, got_idx, a_ref, m, t)
        got = oh.float().numpy().astype(np.float64)
        ref = oracle.sparse_ffn(x, spec, m)
        assert oracle.rel_l2(got, ref) <= (TOL_BF16_F32OUT if dtype == torch.float32 else TOL_BF16)
        assert np.array_equal(got_idx, idx_d)
        assert oracle.rel_l2(got, out_d) <= tol
