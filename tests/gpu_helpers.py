"""Helpers for the GPU parity tests: run the CUDA path through the C ABI and read results back."""
from __future__ import annotations

import numpy as np
import torch

import oracle
from contextual_sparsity_ffn_b200 import binding as cs

DEV = "cuda"


def dev_layer(spec) -> cs.FFNLayer:
    return cs.FFNLayer.from_spec(spec, DEV)


def dev(a) -> torch.Tensor:
    return cs.to_device(a, DEV)


def run_gate(layer: cs.FFNLayer, x_np: np.ndarray, t: float, ws=None, cand=None):
    """csffn_gate_mask on x (numpy [B, d] operand). Returns (idx, a_val [B, count], buffers)."""
    x = dev(x_np if x_np.ndim == 2 else x_np[None, :])
    B = x.shape[0]
    idx = torch.full((layer.h,), -1, dtype=torch.int32, device=DEV)
    count = torch.full((1,), -7, dtype=torch.int32, device=DEV)
    a_val = torch.zeros(max(B, 1), layer.h, dtype=torch.float32, device=DEV)
    if ws is None:
        ws = cs.new_workspace(layer, max(B, 1))
    cand_idx = cand_count = None
    if cand is not None:
        cand_idx, cand_count = cand
    cs.gate_mask(layer, x, t, idx, count, a_val, ws, cand_idx=cand_idx, cand_count=cand_count)
    assert cs.check_status(ws) == 0
    n = int(count.item())
    return (idx[:n].cpu().numpy(), a_val[:B, :n].cpu().numpy().astype(np.float64),
            dict(x=x, idx=idx, count=count, a_val=a_val, ws=ws, n=n))


def run_sparse(layer: cs.FFNLayer, bufs: dict, out_dtype=torch.float32, out_mode=None, out=None):
    B = bufs["x"].shape[0]
    if out is None:
        out = torch.full((B, layer.d), float("nan"), dtype=out_dtype, device=DEV)
    cs.sparse_ffn_forward(layer, bufs["x"], bufs["idx"], bufs["count"], bufs["a_val"], out, bufs["ws"],
                          out_mode=out_mode)
    assert cs.check_status(bufs["ws"]) == 0
    return out.float().cpu().numpy().astype(np.float64)


def run_dense(layer: cs.FFNLayer, x_np: np.ndarray, out_dtype=torch.float32, ws=None):
    x = dev(x_np if x_np.ndim == 2 else x_np[None, :])
    B = x.shape[0]
    if ws is None:
        ws = cs.new_workspace(layer, B)
    out = torch.full((B, layer.d), float("nan"), dtype=out_dtype, device=DEV)
    cs.dense_ffn_forward(layer, x, out, ws)
    assert cs.check_status(ws) == 0
    return out.float().cpu().numpy().astype(np.float64)


def token_masks(idx: np.ndarray, a_val: np.ndarray, h: int) -> np.ndarray:
    """Per-token keep masks [B, h] from the union index list and per-token values (t >= 0)."""
    m = np.zeros((a_val.shape[0], h), dtype=bool)
    m[:, idx] = a_val != 0.0
    return m


def band_rows(a_ref: np.ndarray, t: float, rel: float = 1e-3) -> np.ndarray:
    """Neurons with some token's |a| within rel*t of t: their membership may legitimately differ."""
    return (np.abs(np.abs(a_ref) - t) < rel * abs(t)).any(axis=0)


def assert_index_list(idx: np.ndarray, h: int) -> None:
    assert idx.dtype == np.int32
    assert np.all(idx >= 0) and np.all(idx < h)
    assert np.all(np.diff(idx) > 0), "indices must be unique and ascending"


def check_values(a_val, idx, a_ref, m, t, atol_rel=1e-6):
    """a_val against the oracle's activations, element by element: a where the token keeps the row,
    0 where it rejects it; the per-token masks agree with the oracle's outside the band.  atol_rel
    scales the absolute tolerance by the largest |a| (1e-6 for fp32 sums of one row in order; the
    tensor-core path adds 64-element partial sums, a few times that)."""
    tb = np.abs(np.abs(a_ref) - t) < 1e-3 * abs(t)
    assert np.array_equal(m[~tb], oracle.cats_mask(a_ref, t)[~tb])
    np.testing.assert_allclose(a_val, np.where(m, a_ref, 0.0)[:, idx], rtol=1e-4,
                               atol=atol_rel * np.abs(a_ref).max())
