"""CPU oracle for the contextually sparse gated FFN at decode time.

TEST INFRASTRUCTURE ONLY.  Nothing in the product path may import or call
this module: only the tests, ``__graft_entry__.smoke()`` and the
``cpu_baseline`` / ``--impl reference`` legs of ``bench.py`` do.  It shares
no code with the CUDA library.

Every function computes the plain definition in float64 with numpy (matrix
products, the SVD, a Cholesky factorisation and a linear solve are the only
library primitives used), on exactly the operand bits
the GPU receives (bf16 bit patterns as uint16, or float32).  No blocking,
fusion or reordering: the sparse method reaches the same result faster.

Sources (page titles; sections, figures and tables on each):
  [CATS]   "CATS: Contextually-Aware Thresholding for Sparsity in Large
           Language Models", abstract: a new non-linear activation that
           thresholds the gate activations; a custom GPU kernel whose entry
           points fuse the gate GEMV with the compare and a flag-gated GEMV.
  [SVDP]   "SVD Contextual Sparsity Predictors for Fast LLM Inference",
           abstract; Fig. 1 (offline SVD predictors with calibrated per-neuron
           thresholds, run ahead of each FFN block); Fig. 2 (zero threshold
           gives false negatives); Fig. 3 (gate then up run sequentially on the
           predicted-active neurons, ReGLU); Table 3 ("+ Bias calibration").
  [SIRIUS] "Sirius: Contextual Sparsity with Correction for Efficient LLMs",
           abstract, and its summary page, section "Approach": the sparse and
           the full model share weights; the full model verifies a chunk of
           sparse-generated tokens in parallel.

Readings taken where the pages are silent (each one is listed in the design
notes): the CATS threshold applies to the gate output SiLU(z) with strict
``|a| > t``; the quantile is the lower order statistic v_(ceil(s*M)) without
interpolation; t is one scalar per layer pooled over neurons x calibration
vectors; the SVD predictor factors W_gate^T = U S V^T as U_r = U[:, :r] S_r
(stored transposed, [r, d]) and V_r = V[:, :r] ([h, r]), and its data-whitened
variant takes the truncated SVD of L^T W_gate^T with C = X^T X = L L^T over the
calibration rows (plus a small ridge); tau_i is the
per-neuron lower order statistic of the predictor output at q; the gate bias
is an explicit additive vector; RMSNorm has unit gain and eps = 1e-6.
"""
from __future__ import annotations

import math
from fractions import Fraction

import numpy as np

RMS_EPS = 1e-6


def decode(a) -> np.ndarray:
    """Exact float64 value of a stored operand: bf16 bit patterns (uint16) or float32 (operand
    decoding, no passage of the method)."""
    a = np.asarray(a)
    if a.dtype == np.uint16:
        return (a.astype(np.uint32) << np.uint32(16)).view(np.float32).astype(np.float64)
    return a.astype(np.float64)


def silu(z: np.ndarray) -> np.ndarray:
    """SiLU(z) = z * sigmoid(z) = z / (1 + e^{-z}): the SwiGLU gate activation whose output
    [CATS] (abstract) thresholds."""
    with np.errstate(over="ignore"):
        return z / (1.0 + np.exp(-z))


def relu(z: np.ndarray) -> np.ndarray:
    """ReLU(z) = max(z, 0) (the ReGLU gate activation of [SVDP])."""
    return np.maximum(z, 0.0)


def activation(z: np.ndarray, act: str) -> np.ndarray:
    """The layer's gate activation: SiLU ([CATS] abstract, SwiGLU) or ReLU ([SVDP] abstract, ReGLU)."""
    if act == "silu":
        return silu(z)
    if act == "relu":
        return relu(z)
    raise ValueError(act)


def _tokens(x) -> np.ndarray:
    x = decode(x)
    return x[None, :] if x.ndim == 1 else x


def gate_preactivation(x, layer) -> np.ndarray:
    """The gate projection ([CATS] abstract: the gate GEMV; [SVDP] Fig. 3: the gate of the
    predicted neurons): z[b, i] = x_b . W_gate[i, :] + beta_i  ->  [B, h].  beta is the explicit
    per-neuron gate bias of the ReGLU workload (a reading; absent elsewhere)."""
    z = _tokens(x) @ decode(layer.w_gate).T
    if layer.bias is not None:
        z = z + decode(layer.bias)[None, :]
    return z


def gate_activation(x, layer) -> np.ndarray:
    """a = act(z) ([CATS] abstract: the activation that is thresholded): SiLU for SwiGLU, ReLU
    for ReGLU  ->  [B, h]."""
    return activation(gate_preactivation(x, layer), layer.act)


def up_projection(x, layer) -> np.ndarray:
    """The up projection ([CATS] abstract: the flag-gated GEMV reads only the kept rows;
    [SVDP] Fig. 3: up runs after the gate): u[b, i] = x_b . W_up[i, :]  ->  [B, h]."""
    return _tokens(x) @ decode(layer.w_up).T


def down_projection(g: np.ndarray, layer) -> np.ndarray:
    """The down projection over the gated activations ([CATS] abstract; [SVDP] Fig. 3):
    out[b, :] = sum_i g[b, i] * W_down^T[i, :]  ->  [B, d]."""
    return g @ decode(layer.w_down_t)


def dense_ffn(x, layer) -> np.ndarray:
    """Dense gated FFN: out = (act(x W_gate^T + beta) * (x W_up^T)) W_down.

    This is the full model's FFN that verifies a chunk of sparse tokens
    ([SIRIUS] "Approach": sparse and full model share the weights).
    """
    return down_projection(gate_activation(x, layer) * up_projection(x, layer), layer)


def cats_mask(a: np.ndarray, t: float) -> np.ndarray:
    """[CATS] thresholding: neuron i is active for token b iff |a[b, i]| > t (strict)."""
    return np.abs(a) > t


def sparse_ffn(x, layer, mask: np.ndarray) -> np.ndarray:
    """The dense FFN evaluated with the activations outside ``mask`` set to zero ([CATS]
    abstract: sub-threshold activations are zeroed, so their rows contribute nothing).

    ``mask`` is [B, h] (or [h], broadcast over tokens).  This is the result the
    sparse executor must reach by reading only the active rows.
    """
    a = gate_activation(x, layer)
    m = np.asarray(mask, dtype=bool)
    if m.ndim == 1:
        m = np.broadcast_to(m[None, :], a.shape)
    return down_projection(np.where(m, a, 0.0) * up_projection(x, layer), layer)


def cats_ffn(x, layer, t: float) -> tuple:
    """[CATS] sparse FFN at threshold t -> (out [B, d], per-token mask [B, h])."""
    m = cats_mask(gate_activation(x, layer), t)
    return sparse_ffn(x, layer, m), m


def union_mask(mask: np.ndarray) -> np.ndarray:
    """Rows a small batch must read: the union over tokens of the per-token masks -> [h].

    The pages treat one token at a time; the reading for a batch is that the union selects the
    rows that are read while every token keeps its own values."""
    return np.asarray(mask, dtype=bool).reshape(-1, np.shape(mask)[-1]).any(axis=0)


def active_indices(row_mask: np.ndarray) -> np.ndarray:
    """Ascending int32 indices of the set entries of a [h] mask (the index-order reading: the
    pages fix no order)."""
    return np.flatnonzero(np.asarray(row_mask, dtype=bool)).astype(np.int32)


def order_statistic_rank(s: float, m: int) -> int:
    """k = ceil(s * m), clamped to [0, m]: the rank of the lower order statistic that the
    quantile reading of the calibrated threshold ([CATS] abstract; [SVDP] Fig. 1) selects.

    s is first taken at float32 precision (the type the library interface
    carries), then the product is evaluated exactly; 0.9 of 50 values is 45.
    """
    k = math.ceil(Fraction(float(np.float32(s))) * m)
    return min(max(k, 0), m)


def calibrate_global(x_cal, layer, s: float) -> float:
    """One CATS threshold per layer ([CATS] abstract: a threshold set for a target sparsity):
    the s-quantile of |a| pooled over calibration set x neurons.

    M = N*h values |a|, sorted ascending; k = ceil(s*M); t = v_(k) (1-indexed),
    t = 0 when k = 0.  On the calibration set #{|a| <= t} >= k, with equality
    when no ties occur.
    """
    v = np.sort(np.abs(gate_activation(x_cal, layer)).ravel())
    k = order_statistic_rank(s, v.size)
    return 0.0 if k == 0 else float(v[k - 1])


def svd_factors(w_gate, r: int) -> tuple:
    """[SVDP] abstract / Fig. 1: rank-r truncated SVD of the gate projection.

    The gate maps a row vector x to x W_gate^T, so the projection matrix is
    W_gate^T (d x h) = U S V^T.  Returns (U_r^T [r, d] = (U[:, :r] S_r)^T,
    V_r [h, r] = V[:, :r]) in float64; x U_r V_r^T approximates x W_gate^T.
    """
    u, s, vt = np.linalg.svd(decode(w_gate).T, full_matrices=False)
    return (u[:, :r] * s[None, :r]).T.copy(), vt[:r, :].T.copy()


WHITEN_RIDGE = 1e-6


def svd_factors_whitened(w_gate, r: int, x_cal, ridge: float = WHITEN_RIDGE) -> tuple:
    """[SVDP] abstract ("truncation-aware" SVD) and Table 3 ("+ Data whitening"): the rank-r
    factors of W_gate^T that best reproduce the gate pre-activations of the calibration inputs.

    Reading (the pages name the step but print no formula): among rank-r d x h matrices M,
    minimise ||X (W_gate^T - M)||_F over the calibration rows X [N, d].  With
    C = X^T X + lambda I = L L^T (Cholesky; lambda = ridge * trace(X^T X) / d keeps C
    definite when N < d), ||X A||_F^2 = ||L^T A||_F^2 up to the ridge, so the optimum is the
    truncated SVD of the whitened matrix, L^T W_gate^T = U S V^T, mapped back:
    M = L^{-T} U_r S_r V_r^T.  Returns (U_r^T [r, d] = (L^{-T} U[:, :r] S_r)^T, V_r [h, r]) in
    float64, the same layout as svd_factors; the predictor is unchanged (p = x U_r V_r^T + beta).
    """
    xs = _tokens(x_cal)
    c = xs.T @ xs
    d = c.shape[0]
    c = c + (ridge * np.trace(c) / d) * np.eye(d)
    low = np.linalg.cholesky(c)  # C = L L^T, L lower triangular
    u, s, vt = np.linalg.svd(low.T @ decode(w_gate).T, full_matrices=False)
    u_r = np.linalg.solve(low.T, u[:, :r] * s[None, :r])  # L^{-T} U_r S_r
    return u_r.T.copy(), vt[:r, :].T.copy()


def predict(x, u_rt, v_r, bias=None) -> np.ndarray:
    """[SVDP] Fig. 1: predictor output p = (x U_r) V_r^T + beta  ->  [B, h]."""
    p = (_tokens(x) @ decode(u_rt).T) @ decode(v_r).T
    if bias is not None:
        p = p + decode(bias)[None, :]
    return p


def calibrate_per_neuron(x_cal, u_rt, v_r, bias, q: float) -> np.ndarray:
    """[SVDP] Fig. 1 / Table 3 "bias calibration": per-neuron thresholds tau [h].

    tau_i = k-th smallest of {p_i(x_n)} over the N calibration vectors,
    k = ceil(q*N); tau_i = -inf when k = 0.  Neuron i is then predicted active
    on at most a (1-q) fraction of the calibration inputs.
    """
    p = np.sort(predict(x_cal, u_rt, v_r, bias), axis=0)
    k = order_statistic_rank(q, p.shape[0])
    if k == 0:
        return np.full(p.shape[1], -np.inf)
    return p[k - 1, :].copy()


def recall_thresholds(p: np.ndarray, z: np.ndarray, recall: float) -> np.ndarray:
    """Per-neuron thresholds that reach a target recall of the truly active set on the calibration
    vectors ([SVDP] Table 3, "+ Bias calibration", and Fig. 2: with a zero threshold the predictor
    misses active neurons; the thresholds are moved per neuron to recover them).  The reading: for
    neuron i, the active calibration vectors are A_i = {n : z_i(x_n) > 0} (m_i of them); c_i =
    ceil(R * m_i) of them must be predicted, so tau_i is the largest value below the c_i-th largest
    of {p_i(x_n) : n in A_i}, and p_i > tau_i holds exactly for the predictor outputs at or above
    it.  tau_i = +inf when c_i = 0 (no active vector, or R = 0): the neuron is never predicted.

    p, z: [N, h]; returns tau [h] in p's precision.
    """
    p = np.asarray(p)
    z = np.asarray(z)
    tau = np.full(p.shape[1], np.inf, dtype=p.dtype)
    for i in range(p.shape[1]):
        act = np.sort(p[z[:, i] > 0, i])
        c = order_statistic_rank(recall, act.size)
        if c > 0:
            tau[i] = np.nextafter(act[act.size - c], -np.inf)
    return tau


def calibrate_per_neuron_recall(x_cal, u_rt, v_r, layer, recall: float) -> np.ndarray:
    """recall_thresholds on the predictor outputs p = (x U_r) V_r^T + beta and the gate
    pre-activations z = x W_gate^T + beta of the calibration vectors x_cal [N, d]."""
    return recall_thresholds(predict(x_cal, u_rt, v_r, layer.bias), gate_preactivation(x_cal, layer), recall)


def predicted_mask(p: np.ndarray, tau: np.ndarray) -> np.ndarray:
    """[SVDP] Fig. 1 and Fig. 2: a neuron is predicted active when its predictor output exceeds
    its calibrated threshold, P = {i : p_i > tau_i} per token -> [B, h]."""
    return p > np.asarray(tau, dtype=np.float64)[None, :]


def reglu_sequential(x, layer, pred_mask: np.ndarray) -> tuple:
    """[SVDP] Fig. 3: gate on the predicted set P, then up/down only on A = {i in P : z_i > 0}.

    Returns (out [B, d], A [B, h]).  ``pred_mask`` is per token [B, h] or [h].
    """
    z = gate_preactivation(x, layer)
    p = np.asarray(pred_mask, dtype=bool)
    if p.ndim == 1:
        p = np.broadcast_to(p[None, :], z.shape)
    a_mask = p & (z > 0.0)
    out = down_projection(np.where(a_mask, z, 0.0) * up_projection(x, layer), layer)
    return out, a_mask


def reglu_parallel(x, layer, pred_mask: np.ndarray) -> tuple:
    """[SVDP] Table 2 caption ("r=1024 parallel") and Table 3 ("Parallel pipeline"): the gate and
    the up projection both run on the predicted set P (neither waits for the other); the down
    projection takes their gated product ReLU(z_i) * u_i, which is zero outside
    A = {i in P : z_i > 0}.  The pages name the pipeline without a formula; this is the reading.

    Returns (out [B, d], A [B, h]).  ``pred_mask`` is per token [B, h] or [h].  The output is the
    sequential pipeline's (the pipelines differ in which rows they read, not in what they compute).
    """
    z = gate_preactivation(x, layer)
    p = np.asarray(pred_mask, dtype=bool)
    if p.ndim == 1:
        p = np.broadcast_to(p[None, :], z.shape)
    g = np.where(p, relu(z) * up_projection(x, layer), 0.0)
    return down_projection(g, layer), p & (z > 0.0)


def rmsnorm(v: np.ndarray, eps: float = RMS_EPS) -> np.ndarray:
    """RMSNorm with unit gain: v / sqrt(mean(v^2) + eps), per row.  The input step of the
    decoder blocks whose FFN shapes [SVDP] Table 12 lists; the pages do not print it (reading:
    unit gain, eps = 1e-6)."""
    v = np.asarray(v, dtype=np.float64)
    return v / np.sqrt(np.mean(v * v, axis=-1, keepdims=True) + eps)


def round_to_bf16(v: np.ndarray) -> np.ndarray:
    """Value of v after rounding to bfloat16 (nearest, ties to even), as float64.

    Done through PyTorch's CPU cast, independently of the input encoder.  The bf16 rounding of the
    FFN input is a reading (the pages run bf16 models but print no rounding step).
    """
    import torch

    t = torch.from_numpy(np.ascontiguousarray(v, dtype=np.float64))
    return t.to(torch.float32).to(torch.bfloat16).to(torch.float64).numpy()


def stack_layer(h: np.ndarray, layer, t=None, mask=None) -> tuple:
    """One residual block of the FFN stack: h + FFN(bf16(RMSNorm(h))) (the decoder block around
    the FFN of the models the pages evaluate; the stack itself is a harness, not a page's method).

    With ``mask`` the FFN is the sparse one on that mask; with ``t`` the CATS
    mask at t; with neither, the dense FFN.  Returns (h_next, xn, mask_used).
    """
    xn = round_to_bf16(rmsnorm(h))
    if mask is None and t is not None:
        mask = cats_mask(gate_activation(xn, layer), t)
    y = dense_ffn(xn, layer) if mask is None else sparse_ffn(xn, layer, mask)
    return np.asarray(h, dtype=np.float64) + y, xn, mask


def sirius_round(x_steps, layer, t: float) -> tuple:
    """[SIRIUS] "Approach", FFN part only: the sparse FFN drafts each of the chunk's
    tokens one at a time, then the dense FFN verifies the whole chunk in one batch.

    Each draft uses only its own token's mask, so the T drafts are evaluated together as T
    independent rows (the batched CATS FFN keeps per-token masks and values).
    Returns (sparse outputs [T, d], dense outputs [T, d], masks [T, h]).
    """
    x = _tokens(x_steps)
    sparse, masks = cats_ffn(x, layer, t)
    return sparse, dense_ffn(x, layer), masks


def round_effective_density(masks: np.ndarray) -> dict:
    """[SIRIUS] "Key results" (effective density) and "Approach" (the full model verifies the
    chunk in parallel), FFN weights only.  The pages give the figure but not its formula; reading:
    weight rows a round reads over the rows T dense decode steps read.

    A draft of token t reads all h rows of W_gate and the W_up and W_down^T rows of its kept set
    (n_t rows each); the verify reads all 3h rows once for the whole chunk; T dense decode steps
    read 3h rows each.  Every draft is counted as accepted (no model, so no rejection: the average
    advance length is T).  ``masks``: the drafts' keep masks [T, h].
    Returns {"neuron_density": mean_t n_t / h, "effective_density": (sum_t (h + 2 n_t) + 3h) / (3 h T)}.
    """
    m = np.asarray(masks, dtype=bool)
    T, h = m.shape
    n = m.sum(axis=1).astype(np.float64)
    return {"neuron_density": float(n.mean() / h),
            "effective_density": float((np.sum(h + 2.0 * n) + 3.0 * h) / (3.0 * h * T))}


def draft_agreement(sparse_out: np.ndarray, dense_out: np.ndarray, proj: np.ndarray) -> dict:
    """Agreement of the sparse drafts with the dense verify over a round ([SIRIUS] "Approach": the
    full model verifies the sparse model's tokens).  Without a language-model head, a fixed matrix
    ``proj`` [d, V] stands in for it (a reading): token t agrees when the arg max over V of
    sparse_t . proj equals that of dense_t . proj (first index on ties).
    Returns {"rel_l2": [T] per-token ||s_t - d_t|| / ||d_t||, "top1": [T] bool}.
    """
    s = np.atleast_2d(np.asarray(sparse_out, dtype=np.float64))
    dn = np.atleast_2d(np.asarray(dense_out, dtype=np.float64))
    r = np.asarray(proj, dtype=np.float64)
    rel = np.linalg.norm(s - dn, axis=1) / np.linalg.norm(dn, axis=1)
    top1 = np.argmax(s @ r, axis=1) == np.argmax(dn @ r, axis=1)
    return {"rel_l2": rel, "top1": top1}


def rel_l2(y, y_ref) -> float:
    """max over vectors of ||y - y_ref||_2 / ||y_ref||_2 (0/0 counts as 0): the parity measure,
    no passage of the method."""
    y = np.atleast_2d(np.asarray(y, dtype=np.float64))
    r = np.atleast_2d(np.asarray(y_ref, dtype=np.float64))
    num = np.linalg.norm(y - r, axis=-1)
    den = np.linalg.norm(r, axis=-1)
    out = np.where(den > 0, num / np.where(den > 0, den, 1.0), np.where(num > 0, np.inf, 0.0))
    return float(out.max()) if out.size else 0.0
