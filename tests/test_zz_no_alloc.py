"""The allocation-free sparse forward (csffn_sparse_ffn_forward_static) against the regular one
and against the CPU oracle.

Some callers cannot allocate device memory at all -- a custom operator whose host framework owns
every allocation, or a loop that must never allocate after start-up -- so they cannot create a
workspace.  The static variant keeps its scratch in a library-owned device array instead.  This
file checks, through the C ABI, that two calls in a row give the same output as the workspace
entry point and as the oracle on the same mask, in every output mode, also when a smaller call
follows a larger one (the array keeps the larger call's contents), and that calls too large for
the array are refused without a launch.  It is named so that pytest collects it last.
"""

import numpy as np
import pytest
import torch

import oracle
from contextual_sparsity_ffn_b200 import synth
from contextual_sparsity_ffn_b200 import binding as cs
from contextual_sparsity_ffn_b200 import _abi

from gpu_helpers import dev_layer, run_gate, token_masks

pytestmark = pytest.mark.gpu

TOL = 1e-4  # max relative L2 per output vector, as the other bf16-layer tests with fp32 outputs
TOL_BF16 = 1e-2  # bf16 outputs


def _static_forward(layer, bufs, out, out_mode=_abi.OUT_F32):
    B = bufs["x"].shape[0]
    return cs.load().csffn_sparse_ffn_forward_static(
        layer.ref(), cs._ptr(bufs["x"]), B, cs._ptr(bufs["idx"]), cs._ptr(bufs["count"]),
        cs._ptr(bufs["a_val"]), cs._ptr(out), out_mode, cs._stream())


def _regular_forward(layer, bufs, out, out_mode=_abi.OUT_F32):
    B = bufs["x"].shape[0]
    ws = bufs["ws"]
    return cs.load().csffn_sparse_ffn_forward(
        layer.ref(), cs._ptr(bufs["x"]), B, cs._ptr(bufs["idx"]), cs._ptr(bufs["count"]),
        cs._ptr(bufs["a_val"]), cs._ptr(out), out_mode, cs._ptr(ws), ws.numel(), cs._stream())


def _check_call(spec, layer, B, s, seed, out_mode):
    """One call of each entry point on the same mask: static == regular, and both == the oracle."""
    x = synth.make_tokens(60, seed, synth.ROLE_EVAL, B, spec.d, "bf16", rms_normalise=True)
    t = float(np.quantile(np.abs(oracle.gate_activation(x, spec)), s))
    idx, a_val, bufs = run_gate(layer, x, t)
    ref_cpu = oracle.sparse_ffn(x, spec, token_masks(idx, a_val, spec.h))
    if out_mode == _abi.OUT_BF16:
        dtype, tol, init = torch.bfloat16, TOL_BF16, None
    else:
        dtype, tol = torch.float32, TOL
        # accumulate: a seeded residual that both entry points add into
        init = torch.from_numpy(np.random.default_rng(seed).standard_normal((B, spec.d)).astype(np.float32)).cuda()
    ref = torch.full((B, spec.d), float("nan"), dtype=dtype, device="cuda")
    got = torch.full((B, spec.d), float("nan"), dtype=dtype, device="cuda")
    if out_mode == _abi.OUT_F32_ACCUMULATE:
        ref.copy_(init)
        got.copy_(init)
    assert _regular_forward(layer, bufs, ref, out_mode) == _abi.OK
    assert _static_forward(layer, bufs, got, out_mode) == _abi.OK
    torch.cuda.synchronize()
    got_np = got.double().cpu().numpy()
    ref_np = ref.double().cpu().numpy()
    if out_mode == _abi.OUT_F32_ACCUMULATE:
        base = init.double().cpu().numpy()
        got_np, ref_np = got_np - base, ref_np - base
    err = oracle.rel_l2(got_np, ref_np)
    assert err <= tol, f"static vs workspace entry point: rel L2 {err:.3e}"
    err_o = oracle.rel_l2(got_np, ref_cpu)
    assert err_o <= tol, f"static vs oracle: rel L2 {err_o:.3e}"


@pytest.mark.parametrize("B,s,out_mode", [(1, 0.5, _abi.OUT_F32), (4, 0.9, _abi.OUT_F32),
                                          (2, 0.7, _abi.OUT_BF16), (3, 0.5, _abi.OUT_F32_ACCUMULATE)])
def test_static_matches_workspace_entry_point_twice(B, s, out_mode):
    spec = synth.llama3_8b_stack_layer(0)
    layer = dev_layer(spec)
    for call in range(2):  # two calls in a row, different tokens: the array keeps stale contents
        _check_call(spec, layer, B, s, call, out_mode)


def test_static_smaller_call_after_larger():
    """A call on a smaller layer and batch right after a larger one reads none of the larger call's
    leftovers (the counters are cleared, the rest is rewritten before it is read)."""
    big = synth.llama3_8b_stack_layer(0)
    _check_call(big, dev_layer(big), 4, 0.5, 7, _abi.OUT_F32)
    small = synth.make_layer(61, 1, 1024, 2000, "bf16")
    _check_call(small, dev_layer(small), 1, 0.5, 8, _abi.OUT_F32)


def test_static_refuses_oversized_calls():
    spec = synth.make_layer(61, 0, 4096, 14336, "bf16")
    layer = dev_layer(spec)
    x = torch.zeros(16, 4096, dtype=torch.bfloat16, device="cuda")
    idx = torch.zeros(14336, dtype=torch.int32, device="cuda")
    count = torch.zeros(1, dtype=torch.int32, device="cuda")
    a_val = torch.zeros(16, 14336, device="cuda")
    out = torch.zeros(16, 4096, device="cuda")
    st = cs.load().csffn_sparse_ffn_forward_static(layer.ref(), cs._ptr(x), 16, cs._ptr(idx), cs._ptr(count),
                                                  cs._ptr(a_val), cs._ptr(out), _abi.OUT_F32, cs._stream())
    assert st == _abi.ERR_UNSUPPORTED_SHAPE
