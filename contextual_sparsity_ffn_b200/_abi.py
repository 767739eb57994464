"""ctypes declarations of libcsffn's C ABI (include/csffn.h).

Loading fails loudly: there is no fallback of any kind when the library is
missing.  Build it with ``python -m contextual_sparsity_ffn_b200.build``.
"""
from __future__ import annotations

import ctypes
import os
import re

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libcsffn.so")
HEADER = os.path.join(os.path.dirname(HERE), "include", "csffn.h")

OK, ERR_INVALID_ARG, ERR_UNSUPPORTED_SHAPE, ERR_ALIGNMENT, ERR_WORKSPACE, ERR_CUDA, ERR_TIMEOUT = range(7)
BF16, F32 = 0, 1
OUT_BF16, OUT_F32, OUT_F32_ACCUMULATE = 0, 1, 2
ACT_SILU, ACT_RELU = 0, 1
CAL_GLOBAL_ABS_ACT, CAL_PER_NEURON_PRED, CAL_PER_NEURON_RECALL = 0, 1, 2
MAX_BATCH = 16


class Layer(ctypes.Structure):
    """csffn_layer."""

    _fields_ = [
        ("d", ctypes.c_int32),
        ("h", ctypes.c_int32),
        ("wdtype", ctypes.c_int32),
        ("act", ctypes.c_int32),
        ("w_gate", ctypes.c_void_p),
        ("w_up", ctypes.c_void_p),
        ("w_down_t", ctypes.c_void_p),
        ("gate_bias", ctypes.c_void_p),
    ]


_P = ctypes.c_void_p
_I = ctypes.c_int
_F = ctypes.c_float
_Z = ctypes.c_size_t
_L = ctypes.POINTER(Layer)

SIGNATURES = {
    "csffn_version": (_I, []),
    "csffn_status_string": (ctypes.c_char_p, [_I]),
    "csffn_workspace_size": (_Z, [_L, _I, _I]),
    "csffn_workspace_init": (_I, [_P, _Z, _P]),
    "csffn_check_status": (_I, [_P, _P]),
    "csffn_gate_mask": (_I, [_L, _P, _I, _F, _P, _P, _P, _P, _P, _P, _Z, _P]),
    "csffn_sparse_ffn_forward": (_I, [_L, _P, _I, _P, _P, _P, _P, _I, _P, _Z, _P]),
    "csffn_dense_ffn_forward": (_I, [_L, _P, _I, _P, _I, _P, _Z, _P]),
    "csffn_cats_ffn_forward": (_I, [_L, _P, _I, _F, _P, _P, _P, _P, _P, _P, _I, _P, _Z, _P]),
    "csffn_cats_ffn_forward_host": (_I, [_L, _P, _I, _F, _P, _P, _P, _P, _I, _P, _Z, _P]),
    "csffn_svd_ffn_forward": (_I, [_L, _P, _I, _I, _P, _P, _P, _F, _P, _P, _P, _P, _I, _P, _Z, _P]),
    "csffn_svd_ffn_forward_parallel": (_I, [_L, _P, _I, _I, _P, _P, _P, _F, _P, _P, _P, _P, _I, _P, _Z, _P]),
    "csffn_predict_lowrank": (_I, [_L, _P, _I, _I, _P, _P, _P, _P, _P, _P, _Z, _P]),
    "csffn_calibrate_workspace_size": (_Z, [_L, _I, _I, _I]),
    "csffn_calibrate_threshold": (_I, [_L, _P, _I, _F, _I, _P, _P, _I, _P, _P, _Z, _P]),
    "csffn_kth_workspace_size": (_Z, []),
    "csffn_kth_smallest": (_I, [_P, ctypes.c_int64, ctypes.c_int64, _P, _P, _Z, _P]),
    "csffn_rmsnorm_bf16": (_I, [_P, _I, _I, _F, _P, _P]),
    "csffn_selftest_timeout": (_I, [_P, _Z, _I, _P]),
    "csffn_sparse_ffn_forward_static": (_I, [_L, _P, _I, _P, _P, _P, _P, _I, _P]),
}

_lib = None


def declared_functions(header: str = HEADER) -> list:
    """Names of the functions include/csffn.h declares."""
    with open(header) as f:
        text = re.sub(r"/\*.*?\*/", "", f.read(), flags=re.S)
    return sorted(set(re.findall(r"\b(csffn_[a-z0-9_]+)\s*\(", text)))


def load(path: str = LIB_PATH) -> ctypes.CDLL:
    """Load libcsffn.so and declare every entry point (cached)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(path):
        raise RuntimeError(f"libcsffn.so is not built ({path}); run python -m contextual_sparsity_ffn_b200.build")
    lib = ctypes.CDLL(path)
    for name, (res, args) in SIGNATURES.items():
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    _lib = lib
    return lib


class CsffnError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        msg = load().csffn_status_string(status).decode()
        super().__init__(f"{where}: csffn status {status} ({msg})")


def check(status: int, where: str) -> None:
    if status != OK:
        raise CsffnError(status, where)
