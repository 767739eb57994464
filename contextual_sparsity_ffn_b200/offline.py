"""Offline stage of the SVD sparsity predictor: the low-rank factors of a layer's gate projection.

"SVD Contextual Sparsity Predictors for Fast LLM Inference", Fig. 1: before decoding, each FFN
layer gets a predictor built from a truncated SVD of its gate projection; the abstract calls the
SVD "truncation-aware", and Table 3 ablates naive SVD against "+ Data whitening".  This module
builds both kinds of factors once per layer on the host side (float64 torch linear algebra on
the weights' device); the decode path then only reads them (csffn_predict_lowrank,
csffn_svd_ffn_forward, and csffn_calibrate_threshold for the per-neuron thresholds).

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
