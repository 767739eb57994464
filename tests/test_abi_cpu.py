"""C ABI checks that need no GPU: the library loads, exports every declared symbol, and rejects bad
arguments on the host before any CUDA call (fake, never-dereferenced device pointers)."""
import ctypes

import pytest

from contextual_sparsity_ffn_b200 import _abi
from contextual_sparsity_ffn_b200.build import build

FAKE = 0x7F0000000000  # 16-byte aligned, never dereferenced: every case below fails validation first
BIG = 1 << 40


@pytest.fixture(scope="module")
def lib():
    build()
    return _abi.load()


def layer(d=4096, h=11008, wdtype=_abi.BF16, act=_abi.ACT_SILU, bias=None):
    return _abi.Layer(d, h, wdtype, act, FAKE, FAKE + 0x1000, FAKE + 0x2000, bias)


def P(v):
    return ctypes.c_void_p(v)


def test_exports_every_declared_symbol(lib):
    names = _abi.declared_functions()
    assert len(names) >= 15
    for n in names:
        assert hasattr(lib, n), n
        assert n in _abi.SIGNATURES, f"binding does not declare {n}"
    assert lib.csffn_version() == 1


def test_status_strings(lib):
    for code in range(7):
        assert lib.csffn_status_string(code)
    assert lib.csffn_status_string(99) == b"unknown status"


def test_workspace_size(lib):
    L = layer()
    assert lib.csffn_workspace_size(ctypes.byref(L), 1, 0) > 0
    assert lib.csffn_workspace_size(ctypes.byref(L), 16, 1024) > lib.csffn_workspace_size(ctypes.byref(L), 1, 0)
    assert lib.csffn_workspace_size(ctypes.byref(layer(d=4100)), 1, 0) == 0  # d % 8
    assert lib.csffn_workspace_size(ctypes.byref(L), 17, 0) == 0
    assert lib.csffn_workspace_size(ctypes.byref(L), 0, 0) == 0
    assert lib.csffn_workspace_size(None, 1, 0) == 0


def gate(lib, L, x=FAKE, B=1, t=0.5, cand=None, ccount=None, idx=FAKE, count=FAKE, a_val=FAKE, ws=FAKE, ws_bytes=BIG):
    return lib.csffn_gate_mask(ctypes.byref(L) if L is not None else None, P(x), B, t, P(cand), P(ccount), P(idx),
                               P(count), P(a_val), P(ws), ws_bytes, None)


def test_gate_mask_validation(lib):
    L = layer()
    assert gate(lib, None) == _abi.ERR_INVALID_ARG
    assert gate(lib, layer(d=4100)) == _abi.ERR_ALIGNMENT
    assert gate(lib, layer(d=4)) == _abi.ERR_UNSUPPORTED_SHAPE
    assert gate(lib, layer(h=0)) == _abi.ERR_UNSUPPORTED_SHAPE
    assert gate(lib, layer(wdtype=5)) == _abi.ERR_INVALID_ARG
    assert gate(lib, layer(act=9)) == _abi.ERR_INVALID_ARG
    assert gate(lib, L, B=17) == _abi.ERR_INVALID_ARG
    assert gate(lib, L, B=-1) == _abi.ERR_INVALID_ARG
    assert gate(lib, L, x=0) == _abi.ERR_INVALID_ARG
    assert gate(lib, L, count=0) == _abi.ERR_INVALID_ARG
    assert gate(lib, L, a_val=0) == _abi.ERR_INVALID_ARG
    assert gate(lib, L, cand=FAKE) == _abi.ERR_INVALID_ARG  # list without its count
    assert gate(lib, L, t=float("nan")) == _abi.ERR_INVALID_ARG
    assert gate(lib, L, x=FAKE + 8) == _abi.ERR_ALIGNMENT
    assert gate(lib, L, ws=0) == _abi.ERR_WORKSPACE
    assert gate(lib, L, ws_bytes=100) == _abi.ERR_WORKSPACE
    assert gate(lib, L, ws=FAKE + 4) == _abi.ERR_WORKSPACE
    assert gate(lib, layer(d=16384), B=16) == _abi.ERR_UNSUPPORTED_SHAPE  # tokens exceed shared memory
    bad_w = layer()
    bad_w.w_gate = FAKE + 2
    assert gate(lib, bad_w) == _abi.ERR_ALIGNMENT
    no_w = layer()
    no_w.w_gate = None
    assert gate(lib, no_w) == _abi.ERR_INVALID_ARG


def test_forward_validation(lib):
    L = layer()
    f = lib.csffn_sparse_ffn_forward
    assert f(ctypes.byref(L), P(FAKE), 1, P(FAKE), P(FAKE), P(FAKE), P(FAKE), 7, P(FAKE), BIG, None) == _abi.ERR_INVALID_ARG
    assert f(ctypes.byref(L), P(FAKE), 1, P(0), P(FAKE), P(FAKE), P(FAKE), 1, P(FAKE), BIG, None) == _abi.ERR_INVALID_ARG
    assert f(ctypes.byref(L), P(FAKE), 1, P(FAKE), P(FAKE), P(FAKE), P(FAKE + 4), 1, P(FAKE), BIG, None) == _abi.ERR_ALIGNMENT
    assert f(ctypes.byref(L), P(FAKE), 1, P(FAKE), P(FAKE), P(FAKE), P(FAKE), 1, P(FAKE), 64, None) == _abi.ERR_WORKSPACE
    assert f(ctypes.byref(L), P(FAKE), 0, P(0), P(0), P(0), P(0), 1, P(0), 0, None) == _abi.OK  # empty batch
    g = lib.csffn_dense_ffn_forward
    assert g(ctypes.byref(L), P(FAKE), 1, P(FAKE), 3, P(FAKE), BIG, None) == _abi.ERR_INVALID_ARG
    assert g(ctypes.byref(L), P(0), 1, P(FAKE), 1, P(FAKE), BIG, None) == _abi.ERR_INVALID_ARG
    assert g(ctypes.byref(L), P(FAKE), 1, P(FAKE), 1, P(FAKE), 16, None) == _abi.ERR_WORKSPACE
    assert g(ctypes.byref(L), P(FAKE), 0, P(0), 1, P(0), 0, None) == _abi.OK


def test_predict_validation(lib):
    L = layer(act=_abi.ACT_RELU)
    f = lib.csffn_predict_lowrank
    args = lambda rank=256, u=FAKE, tau=FAKE, ws_bytes=BIG: (ctypes.byref(L), P(FAKE), 1, rank, P(u), P(FAKE),  # noqa
                                                             P(tau), P(FAKE), P(FAKE), P(FAKE), ws_bytes, None)
    assert f(*args(rank=0)) == _abi.ERR_INVALID_ARG
    assert f(*args(rank=5000)) == _abi.ERR_INVALID_ARG
    assert f(*args(rank=100)) == _abi.ERR_ALIGNMENT
    assert f(*args(u=0)) == _abi.ERR_INVALID_ARG
    assert f(*args(tau=0)) == _abi.ERR_INVALID_ARG
    assert f(*args(u=FAKE + 8)) == _abi.ERR_ALIGNMENT
    assert f(*args(ws_bytes=1024)) == _abi.ERR_WORKSPACE


def test_calibrate_validation(lib):
    L = layer()
    f = lib.csffn_calibrate_threshold
    c = lambda n=512, s=0.5, mode=0, rank=0, u=0: f(ctypes.byref(L), P(FAKE), n, s, mode, P(u), P(u), rank,  # noqa
                                                    P(FAKE), P(FAKE), BIG, None)
    assert c(n=0) == _abi.ERR_INVALID_ARG
    assert c(n=9000) == _abi.ERR_INVALID_ARG
    assert c(s=1.5) == _abi.ERR_INVALID_ARG
    assert c(s=-0.1) == _abi.ERR_INVALID_ARG
    assert c(s=float("nan")) == _abi.ERR_INVALID_ARG
    assert c(mode=3) == _abi.ERR_INVALID_ARG
    assert c(mode=1, rank=256, u=0) == _abi.ERR_INVALID_ARG
    assert c(mode=1, rank=100, u=FAKE) == _abi.ERR_ALIGNMENT
    assert lib.csffn_calibrate_workspace_size(ctypes.byref(L), 512, 0, 0) >= 512 * 11008 * 4
    assert lib.csffn_calibrate_workspace_size(ctypes.byref(L), 512, 1, 0) == 0
    assert lib.csffn_calibrate_workspace_size(ctypes.byref(L), 0, 0, 0) == 0
    # the recall mode: the predictor's factors, aligned, and the gate weights (it needs z too)
    assert c(mode=_abi.CAL_PER_NEURON_RECALL, rank=256, u=0) == _abi.ERR_INVALID_ARG
    assert c(mode=_abi.CAL_PER_NEURON_RECALL, rank=100, u=FAKE) == _abi.ERR_ALIGNMENT
    no_gate = layer()
    no_gate.w_gate = None
    assert f(ctypes.byref(no_gate), P(FAKE), 512, 0.9, _abi.CAL_PER_NEURON_RECALL, P(FAKE), P(FAKE), 256, P(FAKE),
             P(FAKE), BIG, None) == _abi.ERR_INVALID_ARG
    assert c(mode=_abi.CAL_PER_NEURON_RECALL, rank=256, u=FAKE, s=1.5) == _abi.ERR_INVALID_ARG
    assert lib.csffn_calibrate_workspace_size(ctypes.byref(L), 512, _abi.CAL_PER_NEURON_RECALL, 0) == 0
    ws_pred = lib.csffn_calibrate_workspace_size(ctypes.byref(L), 512, _abi.CAL_PER_NEURON_PRED, 256)
    ws_recall = lib.csffn_calibrate_workspace_size(ctypes.byref(L), 512, _abi.CAL_PER_NEURON_RECALL, 256)
    assert ws_recall - ws_pred >= 512 * 11008 * 4  # room for z of every calibration vector


def test_kth_rmsnorm_selftest_validation(lib):
    k = lib.csffn_kth_smallest
    ws = lib.csffn_kth_workspace_size()
    assert k(P(FAKE), 10, 11, P(FAKE), P(FAKE), ws, None) == _abi.ERR_INVALID_ARG
    assert k(P(FAKE), 10, 0, P(FAKE), P(FAKE), ws, None) == _abi.ERR_INVALID_ARG
    assert k(P(FAKE), 0, 1, P(FAKE), P(FAKE), ws, None) == _abi.ERR_INVALID_ARG
    assert k(P(FAKE), 10, 1, P(FAKE), P(FAKE), ws - 1, None) == _abi.ERR_WORKSPACE
    r = lib.csffn_rmsnorm_bf16
    assert r(P(FAKE), 1, 0, 1e-6, P(FAKE), None) == _abi.ERR_INVALID_ARG
    assert r(P(0), 1, 64, 1e-6, P(FAKE), None) == _abi.ERR_INVALID_ARG
    assert r(P(FAKE), 1, 64, -1.0, P(FAKE), None) == _abi.ERR_INVALID_ARG
    assert r(P(0), 0, 64, 1e-6, P(0), None) == _abi.OK
    s = lib.csffn_selftest_timeout
    assert s(P(FAKE), BIG, 0, None) == _abi.ERR_INVALID_ARG
    assert s(P(0), BIG, 10, None) == _abi.ERR_WORKSPACE
    assert s(P(FAKE), 16, 10, None) == _abi.ERR_WORKSPACE


def test_one_launch_step_validation(lib):
    """csffn_cats_ffn_forward rejects on the host whatever either of its paths would reject."""
    def call(L=None, x=FAKE, B=1, t=0.5, cand=None, ccount=None, idx=FAKE, count=FAKE, a_val=FAKE, out=FAKE,
             mode=_abi.OUT_F32, ws=FAKE, ws_bytes=BIG):
        L = layer() if L is None else L
        return lib.csffn_cats_ffn_forward(ctypes.byref(L), P(x), B, t, P(cand), P(ccount), P(idx), P(count),
                                          P(a_val), P(out), mode, P(ws), ws_bytes, None)
    assert lib.csffn_cats_ffn_forward(None, P(FAKE), 1, 0.5, None, None, P(FAKE), P(FAKE), P(FAKE), P(FAKE), 1,
                                      P(FAKE), BIG, None) == _abi.ERR_INVALID_ARG
    assert call(B=17) == _abi.ERR_INVALID_ARG
    assert call(mode=9) == _abi.ERR_INVALID_ARG
    assert call(count=0) == _abi.ERR_INVALID_ARG
    assert call(cand=FAKE) == _abi.ERR_INVALID_ARG  # a list without its count
    assert call(ccount=FAKE) == _abi.ERR_INVALID_ARG
    assert call(x=0) == _abi.ERR_INVALID_ARG
    assert call(idx=0) == _abi.ERR_INVALID_ARG
    assert call(a_val=0) == _abi.ERR_INVALID_ARG
    assert call(out=0) == _abi.ERR_INVALID_ARG
    assert call(t=float("nan")) == _abi.ERR_INVALID_ARG
    assert call(x=FAKE + 8) == _abi.ERR_ALIGNMENT
    assert call(out=FAKE + 4) == _abi.ERR_ALIGNMENT
    no_up = layer()
    no_up.w_up = None
    assert call(L=no_up) == _abi.ERR_INVALID_ARG
    bad_down = layer()
    bad_down.w_down_t = FAKE + 0x2002
    assert call(L=bad_down) == _abi.ERR_ALIGNMENT
    assert call(ws=0) == _abi.ERR_WORKSPACE
    assert call(ws_bytes=1 << 20) == _abi.ERR_WORKSPACE
    # shapes neither the one-launch kernels nor the tensor-core path take (d not a multiple of 64) go
    # to the two-call path, whose own limits hold too
    assert call(L=layer(d=16376), B=16) == _abi.ERR_UNSUPPORTED_SHAPE
    assert call(L=layer(d=16376), B=16, idx=0) == _abi.ERR_INVALID_ARG
    assert call(L=layer(d=4100)) == _abi.ERR_ALIGNMENT


def test_host_buffer_step_validation(lib):
    """csffn_cats_ffn_forward_host validates everything before its first copy (the fake host pointers
    below are never read)."""
    def call(L=None, B=1, t=0.5, idx=FAKE, count=FAKE, a_val=FAKE, mode=_abi.OUT_F32, x=FAKE, out=FAKE,
             ws=FAKE, ws_bytes=BIG):
        L = layer() if L is None else L
        return lib.csffn_cats_ffn_forward_host(ctypes.byref(L), P(x), B, t, P(idx), P(count), P(a_val), P(out),
                                               mode, P(ws), ws_bytes, None)
    assert call(mode=_abi.OUT_F32_ACCUMULATE) == _abi.ERR_INVALID_ARG  # no accumulation into host memory
    assert call(B=-1) == _abi.ERR_INVALID_ARG
    assert call(count=0) == _abi.ERR_INVALID_ARG
    assert call(x=0) == _abi.ERR_INVALID_ARG
    assert call(out=0) == _abi.ERR_INVALID_ARG
    assert call(idx=0) == _abi.ERR_INVALID_ARG
    assert call(a_val=0) == _abi.ERR_INVALID_ARG
    assert call(t=float("nan")) == _abi.ERR_INVALID_ARG
    no_gate = layer()
    no_gate.w_gate = None
    assert call(L=no_gate) == _abi.ERR_INVALID_ARG
    assert call(ws_bytes=1 << 20) == _abi.ERR_WORKSPACE  # the staging buffers are part of the workspace
    assert call(L=layer(d=16376), B=16) == _abi.ERR_UNSUPPORTED_SHAPE


def test_predictor_step_validation(lib):
    L = layer(act=_abi.ACT_RELU)
    def call(B=1, rank=256, u=FAKE, v=FAKE, tau=FAKE, t=0.0, idx=FAKE, count=FAKE, a_val=FAKE, out=FAKE,
             mode=_abi.OUT_F32, ws=FAKE, ws_bytes=BIG, L=L):
        return lib.csffn_svd_ffn_forward(ctypes.byref(L), P(FAKE), B, rank, P(u), P(v), P(tau), t, P(idx),
                                         P(count), P(a_val), P(out), mode, P(ws), ws_bytes, None)
    assert call(B=17) == _abi.ERR_INVALID_ARG
    assert call(mode=9) == _abi.ERR_INVALID_ARG
    assert call(count=0) == _abi.ERR_INVALID_ARG
    assert call(rank=0) == _abi.ERR_INVALID_ARG
    assert call(rank=5000) == _abi.ERR_INVALID_ARG
    assert call(rank=100) == _abi.ERR_ALIGNMENT  # rank % 8 (bf16)
    assert call(u=0) == _abi.ERR_INVALID_ARG
    assert call(v=0) == _abi.ERR_INVALID_ARG
    assert call(tau=0) == _abi.ERR_INVALID_ARG
    assert call(t=float("nan")) == _abi.ERR_INVALID_ARG
    assert call(v=FAKE + 8) == _abi.ERR_ALIGNMENT
    assert call(B=8) == _abi.ERR_UNSUPPORTED_SHAPE  # the one-launch kernel takes B <= 4
    assert call(ws_bytes=1 << 20) == _abi.ERR_WORKSPACE


def test_static_entry_validation(lib):
    def call(L=None, B=1, x=FAKE, idx=FAKE, count=FAKE, a_val=FAKE, out=FAKE, mode=_abi.OUT_F32):
        L = layer() if L is None else L
        return lib.csffn_sparse_ffn_forward_static(ctypes.byref(L), P(x), B, P(idx), P(count), P(a_val), P(out),
                                                   mode, None)
    assert lib.csffn_sparse_ffn_forward_static(None, P(FAKE), 1, P(FAKE), P(FAKE), P(FAKE), P(FAKE), 1,
                                               None) == _abi.ERR_INVALID_ARG
    assert call(B=17) == _abi.ERR_INVALID_ARG
    assert call(mode=9) == _abi.ERR_INVALID_ARG
    assert call(idx=0) == _abi.ERR_INVALID_ARG
    assert call(out=FAKE + 4) == _abi.ERR_ALIGNMENT
    assert call(L=layer(d=4100)) == _abi.ERR_ALIGNMENT
    assert call(B=8) == _abi.ERR_UNSUPPORTED_SHAPE  # scratch holds B <= 4 at d = 4096
    assert call(L=layer(d=8192), B=4) == _abi.ERR_UNSUPPORTED_SHAPE
