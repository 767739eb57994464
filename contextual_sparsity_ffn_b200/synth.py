"""Seeded synthetic inputs for the contextually sparse FFN workloads.

This module is shared by the callers of the CUDA path and by the CPU oracle,
so it deliberately holds none of the method's arithmetic: only random draws,
the RMS normalisation that the input recipe applies to token vectors, and the
round-to-nearest-even encoding of float32 values into bfloat16 bit patterns
(the stored operand format).  Every stream is a numpy PCG64 generator seeded
with ``SeedSequence([workload, layer, role])``.

Workloads (shapes follow the models the pages evaluate: LLaMA-2-7B has hidden
size 4096 and intermediate size 11008, Mistral/LLaMA-3-8B 4096/14336 -- "SVD
Contextual Sparsity Predictors for Fast LLM Inference", Table 12):

  0  tiny SwiGLU, fp32, d=256, h=688, 16 decode tokens, 256 calibration vectors
  1  LLaMA-2-7B-shaped SwiGLU, bf16, d=4096, h=11008, 512 calibration vectors
  2  ReGLU with a per-neuron negative gate bias, bf16, d=4096, h=11008
  3  32-layer LLaMA-3-8B-shaped SwiGLU stack, bf16, d=4096, h=14336
  4  LLaMA-3-70B-shaped SwiGLU, bf16, d=8192, h=28672
"""
from __future__ import annotations

from dataclasses import dataclass
from typing import Optional

import numpy as np

ROLE_GATE, ROLE_UP, ROLE_DOWN, ROLE_BIAS = 0, 1, 2, 3
ROLE_CALIB, ROLE_EVAL = 10, 11

WEIGHT_STD = 0.02


def generator(workload: int, layer: int, role: int) -> np.random.Generator:
    return np.random.Generator(np.random.PCG64(np.random.SeedSequence([workload, layer, role])))


def bf16_bits(a: np.ndarray) -> np.ndarray:
    """Round float32 values to bfloat16 (nearest, ties to even); return the bits as uint16.

    Inputs are finite by contract.
    """
    u = np.ascontiguousarray(a, dtype=np.float32).view(np.uint32).astype(np.uint64)
    r = (u + 0x7FFF + ((u >> 16) & 1)) >> 16
    return r.astype(np.uint16)


@dataclass
class LayerSpec:
    """One gated FFN layer as stored for both sides.

    ``w_gate`` and ``w_up`` are [h, d] (row i = neuron i's input weights);
    ``w_down_t`` is [h, d] (row i = neuron i's output weights, i.e. the down
    projection transposed).  bf16 operands are uint16 bit arrays, fp32 ones
    float32 arrays.  ``bias`` is an optional float32 [h] gate bias.
    """

    d: int
    h: int
    dtype: str  # "bf16" | "f32"
    act: str  # "silu" | "relu"
    w_gate: np.ndarray
    w_up: np.ndarray
    w_down_t: np.ndarray
    bias: Optional[np.ndarray] = None


def _weights(workload: int, layer: int, role: int, h: int, d: int, dtype: str) -> np.ndarray:
    w = generator(workload, layer, role).standard_normal((h, d), dtype=np.float32)
    w *= np.float32(WEIGHT_STD)
    return bf16_bits(w) if dtype == "bf16" else w


def make_layer(workload: int, layer: int, d: int, h: int, dtype: str, act: str = "silu",
               bias_mean_std: Optional[tuple] = None) -> LayerSpec:
    """Weights i.i.d. N(0, 0.02^2); optional gate bias i.i.d. N(mean, std^2) in float32."""
    bias = None
    if bias_mean_std is not None:
        mean, std = bias_mean_std
        bias = generator(workload, layer, ROLE_BIAS).normal(mean, std, size=h).astype(np.float32)
    return LayerSpec(d=d, h=h, dtype=dtype, act=act,
                     w_gate=_weights(workload, layer, ROLE_GATE, h, d, dtype),
                     w_up=_weights(workload, layer, ROLE_UP, h, d, dtype),
                     w_down_t=_weights(workload, layer, ROLE_DOWN, h, d, dtype),
                     bias=bias)


def make_tokens(workload: int, layer: int, role: int, n: int, d: int, dtype: str,
                rms_normalise: bool) -> np.ndarray:
    """n token vectors x ~ N(0, 1), optionally scaled to unit root-mean-square per vector."""
    x = generator(workload, layer, role).standard_normal((n, d))
    if rms_normalise:
        x = x / np.sqrt(np.mean(x * x, axis=1, keepdims=True))
    x = x.astype(np.float32)
    return bf16_bits(x) if dtype == "bf16" else x


# --- the five workloads -----------------------------------------------------------------

def tiny_swiglu() -> tuple:
    """Workload 0: (layer, eval tokens [16, 256] f32, calibration [256, 256] f32)."""
    d, h = 256, 688
    layer = make_layer(0, 0, d, h, "f32", "silu")
    x = make_tokens(0, 0, ROLE_EVAL, 16, d, "f32", rms_normalise=False)
    xc = make_tokens(0, 0, ROLE_CALIB, 256, d, "f32", rms_normalise=False)
    return layer, x, xc


def llama2_7b_swiglu(layer_id: int = 0, n_eval: int = 1, n_calib: int = 512) -> tuple:
    """Workload 1: (layer, eval tokens [n_eval, 4096] bf16, calibration [n_calib, 4096] bf16)."""
    d, h = 4096, 11008
    layer = make_layer(1, layer_id, d, h, "bf16", "silu")
    x = make_tokens(1, layer_id, ROLE_EVAL, n_eval, d, "bf16", rms_normalise=True)
    xc = make_tokens(1, layer_id, ROLE_CALIB, n_calib, d, "bf16", rms_normalise=True)
    return layer, x, xc


def reglu_bias_sigma(d: int) -> float:
    """Std of x.W_gate[i] for unit-RMS x and N(0, 0.02^2) weights: 0.02 * sqrt(d)."""
    return WEIGHT_STD * float(np.sqrt(d))


def reglu_sparse(layer_id: int = 0, d: int = 4096, h: int = 11008, n_eval: int = 1,
                 n_calib: int = 512) -> tuple:
    """Workload 2: ReGLU layer whose gate carries a per-neuron offset N(-1.5 s, (0.5 s)^2)."""
    s = reglu_bias_sigma(d)
    layer = make_layer(2, layer_id, d, h, "bf16", "relu", bias_mean_std=(-1.5 * s, 0.5 * s))
    x = make_tokens(2, layer_id, ROLE_EVAL, n_eval, d, "bf16", rms_normalise=True)
    xc = make_tokens(2, layer_id, ROLE_CALIB, n_calib, d, "bf16", rms_normalise=True)
    return layer, x, xc


def sparse_qwen2_reglu(layer_id: int = 0, n_eval: int = 1, n_calib: int = 512) -> tuple:
    """Workload 5: ReGLU layer of the SparseQwen2-7B FFN shape (d 3584, h 18944), gate offsets as in
    workload 2: (layer, eval tokens bf16 unit RMS, calibration tokens)."""
    d, h = 3584, 18944
    s = reglu_bias_sigma(d)
    layer = make_layer(5, layer_id, d, h, "bf16", "relu", bias_mean_std=(-1.5 * s, 0.5 * s))
    x = make_tokens(5, layer_id, ROLE_EVAL, n_eval, d, "bf16", rms_normalise=True)
    xc = make_tokens(5, layer_id, ROLE_CALIB, n_calib, d, "bf16", rms_normalise=True)
    return layer, x, xc


def llama3_8b_stack_layer(layer_id: int) -> LayerSpec:
    """Workload 3: one of the 32 LLaMA-3-8B-shaped SwiGLU layers."""
    return make_layer(3, layer_id, 4096, 14336, "bf16", "silu")


def llama3_8b_stack_tokens(n: int, role: int = ROLE_EVAL) -> np.ndarray:
    """Workload 3 residual-stream inputs: n vectors N(0,1), unit RMS, kept as float32."""
    return make_tokens(3, 0, role, n, 4096, "f32", rms_normalise=True)


def llama3_70b_swiglu(n_eval: int = 16, n_calib: int = 512) -> tuple:
    """Workload 4: (layer, 16 decode tokens bf16 not normalised, calibration bf16)."""
    d, h = 8192, 28672
    layer = make_layer(4, 0, d, h, "bf16", "silu")
    x = make_tokens(4, 0, ROLE_EVAL, n_eval, d, "bf16", rms_normalise=False)
    xc = make_tokens(4, 0, ROLE_CALIB, n_calib, d, "bf16", rms_normalise=False)
    return layer, x, xc
