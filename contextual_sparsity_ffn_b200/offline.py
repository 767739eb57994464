"""Offline stage of the SVD sparsity predictor: the low-rank factors of a layer's gate projection.

"SVD Contextual Sparsity Predictors for Fast LLM Inference", Fig. 1: before decoding, each FFN
layer gets a predictor built from a truncated SVD of its gate projection; the abstract calls the
SVD "truncation-aware", and Table 3 ablates naive SVD against "+ Data whitening".  This module
builds both kinds of factors once per layer on the host side (float64 torch linear algebra on
the weights' device); the decode path then only reads them (csffn_predict_lowrank,
csffn_svd_ffn_forward, and csffn_calibrate_threshold for the per-neuron thresholds).
save_artefacts / load_artefacts keep a layer's offline results (thresholds and factors) on disk.

Layout, as the C entry points take it: the gate maps a token row x to x W_gate^T with
W_gate [h, d] neuron-major, and the predictor computes p = (x U_r) V_r^T + beta with
U_r^T stored as u_rt [r, d] and V_r as v_r [h, r].

* Naive: W_gate^T = U S V^T, U_r = U[:, :r] S_r, V_r = V[:, :r]; U_r V_r^T is the best rank-r
  approximation of W_gate^T in the Frobenius norm.
* Data-whitened: the rank-r M minimising ||X (W_gate^T - M)||_F over calibration token rows
  X [N, d], i.e. the factors that best reproduce the gate pre-activations the layer actually
  sees.  With C = X^T X + lambda I = L L^T (Cholesky), ||X A||_F = ||L^T A||_F up to the ridge,
  so M is the truncated SVD of L^T W_gate^T mapped back by L^{-T}.  lambda = ridge * trace(X^T X)
  / d keeps C definite when N < d; with N >= d the ridge changes the factors only slightly.
"""
from __future__ import annotations

from typing import Optional, Tuple

import numpy as np
import torch

DEFAULT_RIDGE = 1e-6


def svd_predictor_factors(w_gate: torch.Tensor, rank: int, x_cal: Optional[torch.Tensor] = None,
                          ridge: float = DEFAULT_RIDGE,
                          out_dtype: Optional[torch.dtype] = None) -> Tuple[torch.Tensor, torch.Tensor]:
    """Rank-`rank` predictor factors (u_rt [rank, d], v_r [h, rank]) of W_gate [h, d].

    x_cal: calibration token rows [N, d] for the data-whitened factors; None gives the naive
    truncated SVD.  The factorisation runs in float64 on w_gate's device; the factors come back
    contiguous in out_dtype (default: w_gate's dtype, so bf16 weights give bf16 factors).
    Raises ValueError for a rank outside 1 .. min(h, d) or mismatched shapes.
    """
    if w_gate.dim() != 2:
        raise ValueError("w_gate must be [h, d]")
    h, d = w_gate.shape
    if not 1 <= rank <= min(h, d):
        raise ValueError(f"rank must be in 1 .. {min(h, d)}")
    out_dtype = out_dtype or w_gate.dtype
    wt = w_gate.to(torch.float64).T  # W_gate^T [d, h]
    if x_cal is None:
        u, s, vh = torch.linalg.svd(wt, full_matrices=False)
        u_r = u[:, :rank] * s[:rank]
    else:
        if x_cal.dim() != 2 or x_cal.shape[1] != d:
            raise ValueError("x_cal must be [N, d]")
        xs = x_cal.to(device=wt.device, dtype=torch.float64)
        c = xs.T @ xs
        c.diagonal().add_(ridge * torch.trace(c) / d)
        low = torch.linalg.cholesky(c)  # C = L L^T
        u, s, vh = torch.linalg.svd(low.T @ wt, full_matrices=False)
        # U_r = L^{-T} (U[:, :r] S_r): a solve with the upper-triangular L^T
        u_r = torch.linalg.solve_triangular(low.T, u[:, :rank] * s[:rank], upper=True)
    u_rt = u_r.T.to(out_dtype).contiguous()
    v_r = vh[:rank, :].T.to(out_dtype).contiguous()
    return u_rt, v_r


# ------------------------------------------------------------------------------ artefacts on disk

def save_artefacts(path: str, **tensors: torch.Tensor) -> None:
    """Write a layer's offline artefacts (e.g. t, tau, u_rt, v_r) to one .npz file, bit for bit.

    bf16 tensors are stored as their uint16 bit patterns (numpy has no bf16) with the dtype
    recorded beside them, so load_artefacts gives back identical bits.  Calibration and the SVD
    run once per model; a decode process reloads their results instead of repeating them.
    """
    arrays = {}
    for name, t in tensors.items():
        if not isinstance(t, torch.Tensor):
            raise TypeError(f"{name} is not a tensor")
        c = t.detach().cpu().contiguous()
        if c.dtype == torch.bfloat16:
            arrays[name] = c.view(torch.int16).numpy().view(np.uint16)
            arrays["__dtype__" + name] = np.array("bfloat16")
        else:
            arrays[name] = c.numpy()
            arrays["__dtype__" + name] = np.array(str(c.dtype).replace("torch.", ""))
    with open(path, "wb") as f:
        np.savez(f, **arrays)


def load_artefacts(path: str, device="cpu") -> dict:
    """Read a file written by save_artefacts: {name: tensor} with the saved dtypes and bits."""
    out = {}
    with np.load(path, allow_pickle=False) as z:
        for name in z.files:
            if name.startswith("__dtype__"):
                continue
            dt = str(z["__dtype__" + name])
            a = z[name]
            if dt == "bfloat16":
                t = torch.from_numpy(a.view(np.int16).copy()).view(torch.bfloat16)
            else:
                t = torch.from_numpy(a.copy())
                if str(t.dtype).replace("torch.", "") != dt:
                    raise ValueError(f"{name}: stored as {a.dtype}, recorded as {dt}")
            out[name] = t.to(device)
    return out
