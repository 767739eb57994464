"""Thin torch-facing binding of libcsffn: argument marshalling only.

Every function takes CUDA tensors, passes their device pointers and the
current CUDA stream to the C entry point of the same name, and raises
``CsffnError`` on a non-zero status.  No arithmetic of the method happens
here; PyTorch only provides device memory and streams.
"""
from __future__ import annotations

import ctypes
from dataclasses import dataclass, field
from typing import Optional

import numpy as np
import torch

from . import _abi
from ._abi import CsffnError, check, load  # noqa: F401

TORCH_DTYPE = {_abi.BF16: torch.bfloat16, _abi.F32: torch.float32}


def _ptr(t: Optional[torch.Tensor]):
    if t is None:
        return None
    if not t.is_cuda:
        raise ValueError("csffn takes CUDA tensors")
    if not t.is_contiguous():
        raise ValueError("csffn takes contiguous tensors")
    return ctypes.c_void_p(t.data_ptr())


def _stream(stream=None):
    s = stream if stream is not None else torch.cuda.current_stream()
    return ctypes.c_void_p(s.cuda_stream)


@dataclass
class FFNLayer:
    """Device copy of one gated FFN layer plus the csffn_layer struct pointing at it."""

    w_gate: torch.Tensor
    w_up: torch.Tensor
    w_down_t: torch.Tensor
    act: int
    bias: Optional[torch.Tensor] = None
    c: _abi.Layer = field(default=None, repr=False)

    def __post_init__(self):
        h, d = self.w_gate.shape
        wdtype = _abi.BF16 if self.w_gate.dtype == torch.bfloat16 else _abi.F32
        self.c = _abi.Layer(d, h, wdtype, self.act, self.w_gate.data_ptr(), self.w_up.data_ptr(),
                            self.w_down_t.data_ptr(), self.bias.data_ptr() if self.bias is not None else None)

    @property
    def d(self) -> int:
        return self.c.d

    @property
    def h(self) -> int:
        return self.c.h

    @property
    def wdtype(self) -> int:
        return self.c.wdtype

    @property
    def dtype(self) -> torch.dtype:
        return TORCH_DTYPE[self.c.wdtype]

    @classmethod
    def from_spec(cls, spec, device="cuda") -> "FFNLayer":
        """Upload a synth.LayerSpec (bf16 bits as uint16, or float32) to the device."""
        def up(a):
            return to_device(a, device)
        act = _abi.ACT_SILU if spec.act == "silu" else _abi.ACT_RELU
        bias = torch.from_numpy(np.ascontiguousarray(spec.bias)).to(device) if spec.bias is not None else None
        return cls(up(spec.w_gate), up(spec.w_up), up(spec.w_down_t), act, bias)

    def ref(self):
        return ctypes.byref(self.c)


def to_device(a: np.ndarray, device="cuda") -> torch.Tensor:
    """numpy operand -> device tensor: uint16 arrays are bf16 bit patterns."""
    a = np.ascontiguousarray(a)
    if a.dtype == np.uint16:
        return torch.from_numpy(a.view(np.int16)).to(device).view(torch.bfloat16)
    return torch.from_numpy(a).to(device)


def to_numpy_bits(t: torch.Tensor) -> np.ndarray:
    """device tensor -> numpy (bf16 as uint16 bit patterns)."""
    t = t.detach().cpu().contiguous()
    if t.dtype == torch.bfloat16:
        return t.view(torch.int16).numpy().view(np.uint16)
    return t.numpy()


# ------------------------------------------------------------------------------ workspace

def workspace_size(layer: FFNLayer, max_batch: int, max_rank: int = 0) -> int:
    n = load().csffn_workspace_size(layer.ref(), max_batch, max_rank)
    if n == 0:
        raise CsffnError(_abi.ERR_INVALID_ARG, "csffn_workspace_size")
    return int(n)


def workspace_init(ws: torch.Tensor, stream=None) -> None:
    check(load().csffn_workspace_init(_ptr(ws), ws.numel() * ws.element_size(), _stream(stream)),
          "csffn_workspace_init")


def new_workspace(layer: FFNLayer, max_batch: int, max_rank: int = 0, device="cuda") -> torch.Tensor:
    ws = torch.empty(workspace_size(layer, max_batch, max_rank), dtype=torch.uint8, device=device)
    workspace_init(ws)
    return ws


def check_status(ws: torch.Tensor, stream=None) -> int:
    """Synchronise and return the device-side status (0 = ok, 6 = a bounded wait timed out)."""
    return int(load().csffn_check_status(_ptr(ws), _stream(stream)))


def _nbytes(t: torch.Tensor) -> int:
    return t.numel() * t.element_size()


# ------------------------------------------------------------------------------ decode path

def gate_mask(layer: FFNLayer, x: torch.Tensor, t: float, idx: torch.Tensor, count: torch.Tensor,
              a_val: torch.Tensor, ws: torch.Tensor, cand_idx: Optional[torch.Tensor] = None,
              cand_count: Optional[torch.Tensor] = None, stream=None) -> None:
    B = x.shape[0] if x.dim() == 2 else 1
    check(load().csffn_gate_mask(layer.ref(), _ptr(x), B, float(t), _ptr(cand_idx), _ptr(cand_count),
                                 _ptr(idx), _ptr(count), _ptr(a_val), _ptr(ws), _nbytes(ws), _stream(stream)),
          "csffn_gate_mask")


def sparse_ffn_forward(layer: FFNLayer, x: torch.Tensor, idx: torch.Tensor, count: torch.Tensor,
                       a_val: torch.Tensor, out: torch.Tensor, ws: torch.Tensor,
                       out_mode: Optional[int] = None, stream=None) -> None:
    B = x.shape[0] if x.dim() == 2 else 1
    if out_mode is None:
        out_mode = _abi.OUT_BF16 if out.dtype == torch.bfloat16 else _abi.OUT_F32
    check(load().csffn_sparse_ffn_forward(layer.ref(), _ptr(x), B, _ptr(idx), _ptr(count), _ptr(a_val),
                                          _ptr(out), out_mode, _ptr(ws), _nbytes(ws), _stream(stream)),
          "csffn_sparse_ffn_forward")


def cats_ffn_forward(layer: FFNLayer, x: torch.Tensor, t: float, idx: torch.Tensor, count: torch.Tensor,
                     a_val: torch.Tensor, out: torch.Tensor, ws: torch.Tensor, out_mode: Optional[int] = None,
                     cand_idx: Optional[torch.Tensor] = None, cand_count: Optional[torch.Tensor] = None,
                     stream=None) -> None:
    B = x.shape[0] if x.dim() == 2 else 1
    if out_mode is None:
        out_mode = _abi.OUT_BF16 if out.dtype == torch.bfloat16 else _abi.OUT_F32
    check(load().csffn_cats_ffn_forward(layer.ref(), _ptr(x), B, float(t), _ptr(cand_idx), _ptr(cand_count),
                                        _ptr(idx), _ptr(count), _ptr(a_val), _ptr(out), out_mode, _ptr(ws),
                                        _nbytes(ws), _stream(stream)),
          "csffn_cats_ffn_forward")


def _host_ptr(t: torch.Tensor):
    if t.is_cuda:
        raise ValueError("csffn host entry points take CPU tensors (pinned for asynchronous copies)")
    if not t.is_contiguous():
        raise ValueError("csffn takes contiguous tensors")
    return ctypes.c_void_p(t.data_ptr())


def cats_ffn_forward_host(layer: FFNLayer, x_host: torch.Tensor, t: float, idx: torch.Tensor,
                          count: torch.Tensor, a_val: torch.Tensor, out_host: torch.Tensor, ws: torch.Tensor,
                          stream=None) -> None:
    """csffn_cats_ffn_forward_host: x_host and out_host are CPU tensors.  Pinned (page-locked)
    tensors are read and written by the step itself over the host link; pageable ones are staged
    through the workspace by copies.  The result is in out_host once the step has completed on the
    stream, and x_host must stay unchanged until then."""
    B = x_host.shape[0] if x_host.dim() == 2 else 1
    out_mode = _abi.OUT_BF16 if out_host.dtype == torch.bfloat16 else _abi.OUT_F32
    check(load().csffn_cats_ffn_forward_host(layer.ref(), _host_ptr(x_host), B, float(t), _ptr(idx), _ptr(count),
                                             _ptr(a_val), _host_ptr(out_host), out_mode, _ptr(ws), _nbytes(ws),
                                             _stream(stream)),
          "csffn_cats_ffn_forward_host")


def dense_ffn_forward(layer: FFNLayer, x: torch.Tensor, out: torch.Tensor, ws: torch.Tensor,
                      out_mode: Optional[int] = None, stream=None) -> None:
    B = x.shape[0] if x.dim() == 2 else 1
    if out_mode is None:
        out_mode = _abi.OUT_BF16 if out.dtype == torch.bfloat16 else _abi.OUT_F32
    check(load().csffn_dense_ffn_forward(layer.ref(), _ptr(x), B, _ptr(out), out_mode, _ptr(ws),
                                         _nbytes(ws), _stream(stream)),
          "csffn_dense_ffn_forward")


def predict_lowrank(layer: FFNLayer, x: torch.Tensor, u_rt: torch.Tensor, v_r: torch.Tensor,
                    tau: torch.Tensor, cand_idx: torch.Tensor, cand_count: torch.Tensor,
                    ws: torch.Tensor, stream=None) -> None:
    B = x.shape[0] if x.dim() == 2 else 1
    rank = u_rt.shape[0]
    check(load().csffn_predict_lowrank(layer.ref(), _ptr(x), B, rank, _ptr(u_rt), _ptr(v_r), _ptr(tau),
                                       _ptr(cand_idx), _ptr(cand_count), _ptr(ws), _nbytes(ws),
                                       _stream(stream)),
          "csffn_predict_lowrank")


def svd_ffn_forward(layer: FFNLayer, x: torch.Tensor, u_rt: torch.Tensor, v_r: torch.Tensor, tau: torch.Tensor,
                    t: float, idx: torch.Tensor, count: torch.Tensor, a_val: torch.Tensor, out: torch.Tensor,
                    ws: torch.Tensor, out_mode: Optional[int] = None, stream=None, parallel: bool = False) -> None:
    """csffn_svd_ffn_forward, or with parallel=True csffn_svd_ffn_forward_parallel (same outputs)."""
    B = x.shape[0] if x.dim() == 2 else 1
    rank = u_rt.shape[0]
    if out_mode is None:
        out_mode = _abi.OUT_BF16 if out.dtype == torch.bfloat16 else _abi.OUT_F32
    name = "csffn_svd_ffn_forward_parallel" if parallel else "csffn_svd_ffn_forward"
    check(getattr(load(), name)(layer.ref(), _ptr(x), B, rank, _ptr(u_rt), _ptr(v_r), _ptr(tau), float(t),
                                _ptr(idx), _ptr(count), _ptr(a_val), _ptr(out), out_mode, _ptr(ws), _nbytes(ws),
                                _stream(stream)),
          name)


def calibrate_workspace_size(layer: FFNLayer, n: int, mode: int, rank: int = 0) -> int:
    s = load().csffn_calibrate_workspace_size(layer.ref(), n, mode, rank)
    if s == 0:
        raise CsffnError(_abi.ERR_INVALID_ARG, "csffn_calibrate_workspace_size")
    return int(s)


def calibrate_threshold(layer: FFNLayer, x_cal: torch.Tensor, target_sparsity: float, mode: int,
                        t_out: torch.Tensor, u_rt: Optional[torch.Tensor] = None,
                        v_r: Optional[torch.Tensor] = None, ws: Optional[torch.Tensor] = None,
                        stream=None) -> None:
    n = x_cal.shape[0]
    rank = u_rt.shape[0] if u_rt is not None else 0
    if ws is None:
        ws = torch.empty(calibrate_workspace_size(layer, n, mode, rank), dtype=torch.uint8, device=x_cal.device)
    check(load().csffn_calibrate_threshold(layer.ref(), _ptr(x_cal), n, float(target_sparsity), mode,
                                           _ptr(u_rt), _ptr(v_r), rank, _ptr(t_out), _ptr(ws), _nbytes(ws),
                                           _stream(stream)),
          "csffn_calibrate_threshold")


def kth_smallest(values: torch.Tensor, k: int, out: torch.Tensor, ws: Optional[torch.Tensor] = None,
                 stream=None) -> None:
    if ws is None:
        ws = torch.empty(int(load().csffn_kth_workspace_size()), dtype=torch.uint8, device=values.device)
    check(load().csffn_kth_smallest(_ptr(values), values.numel(), int(k), _ptr(out), _ptr(ws), _nbytes(ws),
                                    _stream(stream)),
          "csffn_kth_smallest")


def rmsnorm_bf16(h: torch.Tensor, eps: float, xn: torch.Tensor, stream=None) -> None:
    B, d = h.shape
    check(load().csffn_rmsnorm_bf16(_ptr(h), B, d, float(eps), _ptr(xn), _stream(stream)), "csffn_rmsnorm_bf16")


def selftest_timeout(ws: torch.Tensor, spin_limit: int, stream=None) -> None:
    check(load().csffn_selftest_timeout(_ptr(ws), _nbytes(ws), int(spin_limit), _stream(stream)),
          "csffn_selftest_timeout")


# ------------------------------------------------------------------------------ buffers

@dataclass
class DecodeBuffers:
    """Per-layer-shape device buffers of one CATS decode step (batch <= max_batch)."""

    idx: torch.Tensor
    count: torch.Tensor
    a_val: torch.Tensor
    ws: torch.Tensor

    @classmethod
    def new(cls, layer: FFNLayer, max_batch: int, max_rank: int = 0, device="cuda") -> "DecodeBuffers":
        return cls(idx=torch.zeros(layer.h, dtype=torch.int32, device=device),
                   count=torch.zeros(1, dtype=torch.int32, device=device),
                   a_val=torch.zeros(max_batch, layer.h, dtype=torch.float32, device=device),
                   ws=new_workspace(layer, max_batch, max_rank, device))


def cats_decode(layer: FFNLayer, x: torch.Tensor, t: float, out: torch.Tensor, buf: DecodeBuffers,
                out_mode: Optional[int] = None, stream=None, one_launch: bool = True) -> None:
    """One CATS sparse FFN step: the single-launch csffn_cats_ffn_forward, or with
    one_launch=False csffn_gate_mask then csffn_sparse_ffn_forward (same outputs)."""
    if one_launch:
        cats_ffn_forward(layer, x, t, buf.idx, buf.count, buf.a_val, out, buf.ws, out_mode=out_mode, stream=stream)
        return
    gate_mask(layer, x, t, buf.idx, buf.count, buf.a_val, buf.ws, stream=stream)
    sparse_ffn_forward(layer, x, buf.idx, buf.count, buf.a_val, out, buf.ws, out_mode=out_mode, stream=stream)
