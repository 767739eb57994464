"""CUDA path vs the CPU oracle: RMSNorm + residual FFN stack, the Sirius draft/verify round, and
failure detection by bounded device-side waits."""
import numpy as np
import pytest
import torch

import oracle
from contextual_sparsity_ffn_b200 import synth
from contextual_sparsity_ffn_b200 import binding as cs
from contextual_sparsity_ffn_b200 import _abi

from gpu_helpers import dev_layer, run_dense, run_gate, run_sparse, token_masks

pytestmark = pytest.mark.gpu


def test_rmsnorm_bf16():
    h = np.random.default_rng(3).standard_normal((5, 4096)).astype(np.float32) * 3
    xn = torch.empty(5, 4096, dtype=torch.bfloat16, device="cuda")
    cs.rmsnorm_bf16(torch.from_numpy(h).cuda(), 1e-6, xn)
    got = xn.float().cpu().numpy().astype(np.float64)
    ref = oracle.round_to_bf16(oracle.rmsnorm(h.astype(np.float64)))
    ulp = np.abs(ref) * 2.0 ** -7
    assert np.all(np.abs(got - ref) <= ulp + 1e-30)
    assert np.mean(got == ref) > 0.99


@pytest.mark.parametrize("B", [1, 4])
def test_stack_layers(B):
    """Four layers of the 8B-shaped stack: h <- h + FFN(bf16(RMSNorm(h))), CATS at 50%.

    Each layer is checked on the GPU's own input xn and mask; the residual stream is then carried
    on the GPU (accumulate mode), so drift stays in the final end-to-end comparison."""
    n_layers = 4
    hs = synth.llama3_8b_stack_tokens(B)
    h_dev = torch.from_numpy(hs).cuda()
    h_ref = hs.astype(np.float64)
    xn = torch.empty(B, 4096, dtype=torch.bfloat16, device="cuda")
    for li in range(n_layers):
        spec = synth.llama3_8b_stack_layer(li)
        layer = dev_layer(spec)
        cs.rmsnorm_bf16(h_dev, oracle.RMS_EPS, xn)
        xn_np = cs.to_numpy_bits(xn)
        t = float(np.quantile(np.abs(oracle.gate_activation(xn_np, spec)), 0.5))
        idx, a_val, bufs = run_gate(layer, xn_np, t)
        m = token_masks(idx, a_val, spec.h)
        before = h_dev.double().cpu().numpy()
        cs.sparse_ffn_forward(layer, bufs["x"], bufs["idx"], bufs["count"], bufs["a_val"], h_dev, bufs["ws"],
                              out_mode=_abi.OUT_F32_ACCUMULATE)
        delta = h_dev.double().cpu().numpy() - before
        assert oracle.rel_l2(delta, oracle.sparse_ffn(xn_np, spec, m)) <= 1e-4
        h_ref, _, _ = oracle.stack_layer(h_ref, spec, mask=m)
    assert oracle.rel_l2(h_dev.double().cpu().numpy(), h_ref) <= 1e-2


def test_sirius_round_small():
    """16 sparse batch-1 drafts, then one dense verify over the 16-token chunk, same weights."""
    spec = synth.make_layer(58, 0, 2048, 5632, "bf16")
    x = synth.make_tokens(58, 0, synth.ROLE_EVAL, 16, 2048, "bf16", rms_normalise=False)
    t = float(np.quantile(np.abs(oracle.gate_activation(x, spec)), 0.5))
    layer = dev_layer(spec)
    ws = cs.new_workspace(layer, 16)
    masks = []
    outs = []
    for b in range(16):
        idx, a_val, bufs = run_gate(layer, x[b:b + 1], t, ws=ws)
        outs.append(run_sparse(layer, bufs)[0])
        masks.append(token_masks(idx, a_val, spec.h)[0])
    dense = run_dense(layer, x, ws=ws)
    sp_ref, de_ref, m_ref = oracle.sirius_round(x, spec, t)
    assert oracle.rel_l2(dense, de_ref) <= 1e-2
    assert oracle.rel_l2(np.stack(outs), oracle.sparse_ffn(x, spec, np.stack(masks))) <= 1e-4


def test_timeout_is_reported_and_context_survives():
    spec = synth.make_layer(59, 0, 256, 512, "bf16")
    layer = dev_layer(spec)
    ws = cs.new_workspace(layer, 1)
    cs.selftest_timeout(ws, 1000)
    assert cs.check_status(ws) == _abi.ERR_TIMEOUT
    assert cs.check_status(ws) == _abi.OK  # read-and-clear
    cs.workspace_init(ws)
    x = synth.make_tokens(59, 0, synth.ROLE_EVAL, 1, 256, "bf16", rms_normalise=True)
    idx, a_val, bufs = run_gate(layer, x, 0.1, ws=ws)
    out = run_sparse(layer, bufs)
    m = token_masks(idx, a_val, spec.h)
    assert oracle.rel_l2(out, oracle.sparse_ffn(x, spec, m)) <= 1e-4
