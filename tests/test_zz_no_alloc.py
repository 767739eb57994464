"""The allocation-free sparse forward (csffn_sparse_ffn_forward_static) against the regular one.

Some callers cannot allocate device memory at all -- a custom operator whose host framework owns
every allocation, or a loop that must never allocate after start-up -- so they cannot create a
workspace.  The static variant keeps its scratch in a library-owned device array instead.  This
file checks, through the C ABI, that two calls in a row give the same output as the workspace
entry point, and that calls too large for the array are refused without a launch.  It is named
so that pytest collects it last.
"""

import numpy as np
import pytest
import torch

import oracle
from contextual_sparsity_ffn_b200 import synth
from contextual_sparsity_ffn_b200 import binding as cs
from contextual_sparsity_ffn_b200 import _abi

from gpu_helpers import dev_layer, run_gate

pytestmark = pytest.mark.gpu

TOL = 1e-4  # max relative L2 per output vector, as the other bf16-layer tests with fp32 outputs


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


@pytest.mark.parametrize("B,s", [(1, 0.5), (4, 0.9)])
def test_static_matches_workspace_entry_point_twice(B, s):
    spec = synth.llama3_8b_stack_layer(0)
    layer = dev_layer(spec)
    for call in range(2):  # two calls in a row, different tokens: the array keeps stale contents
        x = synth.make_tokens(60, call, synth.ROLE_EVAL, B, spec.d, "bf16", rms_normalise=True)
        t = float(np.quantile(np.abs(oracle.gate_activation(x, spec)), s))
        _, _, bufs = run_gate(layer, x, t)
        ref = torch.full((B, spec.d), float("nan"), device="cuda")
        got = torch.full((B, spec.d), float("nan"), device="cuda")
        assert _regular_forward(layer, bufs, ref) == _abi.OK
        assert _static_forward(layer, bufs, got) == _abi.OK
        torch.cuda.synchronize()
        err = oracle.rel_l2(got.double().cpu().numpy(), ref.double().cpu().numpy())
        assert err <= TOL, f"call {call}: rel L2 {err:.3e}"


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
