"""Compositions of the library's entry points: a residual stack of sparse FFN layers and a Sirius
round (sparse drafts, then the dense verify of the chunk).

These only sequence C-ABI calls (csffn_rmsnorm_bf16, csffn_calibrate_threshold,
csffn_dense_ffn_forward, csffn_cats_ffn_forward); every step of the arithmetic runs in the library.

Stack ("SVD Contextual Sparsity Predictors for Fast LLM Inference", Table 12: the LLaMA-3-8B FFN
shape; the block structure is the plain reading): h <- h + FFN(bf16(RMSNorm(h))) per layer, the
residual h in fp32, the FFN output added in place (CSFFN_OUT_F32_ACCUMULATE).  Each layer's CATS
threshold is calibrated on the calibration vectors carried through the DENSE stack, RMSNorm'd at
that layer.

Sirius round ("SIRIUS : Contexual Sparisty with Correction for Efficient LLMs", "Approach"): the
sparse FFN drafts the chunk's tokens one at a time, then the full FFN (same weights) runs on the
whole chunk at once.
"""
from __future__ import annotations

from dataclasses import dataclass
from typing import List, Optional

import torch

from . import _abi
from . import binding as cs

RMS_EPS = 1e-6
DENSE_CHUNK = 16  # tokens per csffn_dense_ffn_forward call (its batch limit)


def calibrate_stack(layers: List[cs.FFNLayer], h_cal: torch.Tensor, sparsity: float,
                    ws: torch.Tensor, keep_inputs: Optional[dict] = None) -> List[float]:
    """Per-layer CATS thresholds: h_cal [n, d] fp32 (device, updated in place) is carried through the
    dense stack; layer l's threshold is calibrated on bf16(RMSNorm(h_cal)) at that layer.  ws: a
    workspace of the layers' shape for batch 16.  ``keep_inputs``: a dict whose keys are layer
    numbers; each gets that layer's calibration input (bf16 bits on the host), for checks."""
    n, d = h_cal.shape
    xn = torch.empty(n, d, dtype=torch.bfloat16, device=h_cal.device)
    t_dev = torch.zeros(1, device=h_cal.device)
    ts = []
    for layer in layers:
        cs.rmsnorm_bf16(h_cal, RMS_EPS, xn)
        if keep_inputs is not None and len(ts) in keep_inputs:
            keep_inputs[len(ts)] = cs.to_numpy_bits(xn)
        cs.calibrate_threshold(layer, xn, sparsity, _abi.CAL_GLOBAL_ABS_ACT, t_dev)
        ts.append(float(t_dev.item()))
        for b0 in range(0, n, DENSE_CHUNK):
            b1 = min(n, b0 + DENSE_CHUNK)
            cs.dense_ffn_forward(layer, xn[b0:b1], h_cal[b0:b1], ws, out_mode=_abi.OUT_F32_ACCUMULATE)
    return ts


@dataclass
class StackBuffers:
    xn: torch.Tensor        # bf16 [B, d]: the current layer's input
    buf: cs.DecodeBuffers   # idx / count / a_val / workspace of one step


def stack_buffers(layer: cs.FFNLayer, B: int) -> StackBuffers:
    return StackBuffers(xn=torch.empty(B, layer.d, dtype=torch.bfloat16, device="cuda"),
                        buf=cs.DecodeBuffers.new(layer, B))


def sparse_stack(layers: List[cs.FFNLayer], ts: List[float], h: torch.Tensor, sb: StackBuffers,
                 record: Optional[list] = None, counts: Optional[list] = None) -> None:
    """One decode step through the stack: for each layer, xn = bf16(RMSNorm(h)), then
    h += CATS-FFN(xn) by csffn_cats_ffn_forward (accumulate mode).  With ``record`` (a list), each
    layer appends (xn, idx, a_val, h before, h after) copies on the host, for checks; with
    ``counts``, each layer appends the size of its active list (both synchronise every layer)."""
    for layer, t in zip(layers, ts):
        cs.rmsnorm_bf16(h, RMS_EPS, sb.xn)
        before = h.clone() if record is not None else None
        cs.cats_ffn_forward(layer, sb.xn, t, sb.buf.idx, sb.buf.count, sb.buf.a_val, h, sb.buf.ws,
                            out_mode=_abi.OUT_F32_ACCUMULATE)
        if record is not None:
            n = int(sb.buf.count.item())
            B = h.shape[0]
            record.append((cs.to_numpy_bits(sb.xn), sb.buf.idx[:n].cpu().numpy(),
                           sb.buf.a_val[:B, :n].cpu().numpy(), before.cpu().numpy(), h.cpu().numpy()))
        if counts is not None:
            counts.append(int(sb.buf.count.item()))


def dense_stack(layers: List[cs.FFNLayer], h: torch.Tensor, xn: torch.Tensor, ws: torch.Tensor) -> None:
    """The same step with every layer dense: xn = bf16(RMSNorm(h)), h += FFN(xn) by
    csffn_dense_ffn_forward (accumulate mode), batch <= 16."""
    for layer in layers:
        cs.rmsnorm_bf16(h, RMS_EPS, xn)
        cs.dense_ffn_forward(layer, xn, h, ws, out_mode=_abi.OUT_F32_ACCUMULATE)


def sirius_round(layer: cs.FFNLayer, x: torch.Tensor, t: float, sparse_out: torch.Tensor, dense_out: torch.Tensor,
                 buf: cs.DecodeBuffers, ws_dense: torch.Tensor, record: Optional[list] = None) -> None:
    """The FFN work of one Sirius round on a chunk x [T, d]: T one-token sparse steps
    (csffn_cats_ffn_forward, batch 1) into sparse_out [T, d], then one dense forward of the whole
    chunk (csffn_dense_ffn_forward, batch T <= 16) into dense_out [T, d].  With ``record``, each
    draft appends its (idx, a_val) on the host."""
    T = x.shape[0]
    for k in range(T):
        cs.cats_ffn_forward(layer, x[k:k + 1], t, buf.idx, buf.count, buf.a_val, sparse_out[k:k + 1], buf.ws)
        if record is not None:
            n = int(buf.count.item())
            record.append((buf.idx[:n].cpu().numpy(), buf.a_val[:1, :n].cpu().numpy()))
    cs.dense_ffn_forward(layer, x, dense_out, ws_dense)


def round_effective_density(counts, h: int) -> float:
    """Weight rows one Sirius round reads over the rows T dense decode steps read (FFN weights): each
    one-token draft reads all h rows of W_gate and the W_up and W_down^T rows of its n_t kept
    neurons, the verify reads the 3 h rows once for the chunk, and every draft counts as accepted.
    ``counts``: the drafts' n_t.  (sum_t (h + 2 n_t) + 3 h) / (3 h T)."""
    T = len(counts)
    return (sum(h + 2.0 * n for n in counts) + 3.0 * h) / (3.0 * h * T)
