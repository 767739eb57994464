#!/usr/bin/env python
"""Benchmark of the contextually sparse FFN decode step on B200.

Workload: LLaMA-2-7B-shaped SwiGLU FFN layer (d=4096, h=11008), bf16 weights, fp32
accumulation, batch-1 decode, CATS threshold calibrated by csffn_calibrate_threshold
on 512 seeded calibration vectors at 50% target sparsity (70% and 90% and the dense
path of the same library are measured too and reported under "detail").

A step is one CATS decode of one layer through csffn_cats_ffn_forward: gate GEMV + SiLU +
threshold and the gathered up and down projections of the kept rows in a streaming kernel
(cats_ring_kernel), then the sum of the CTAs' partial outputs and the compaction of the active list
in a short finishing kernel (ring_finish_kernel) launched as its programmatic dependent: two
launches per step.  The two-call path (csffn_gate_mask then csffn_sparse_ffn_forward, three
kernels) is reported under "detail", with 70% and 90%, the dense path, the SVD-predictor ReGLU
step, the 32-layer LLaMA-3-8B-shaped stack at batch 1/4/16 and the LLaMA-3-70B-shaped Sirius round.
The timed steps rotate over 8 distinct layer weight sets (2.2 GB, many times the 126 MB L2)
so no step reads weights that an earlier step left in L2.  K steps are captured in one
CUDA graph and timed with CUDA events on the capture stream.

With N > 1 (torchrun) every rank runs an independent replica (the decode step has no
exchange step); the time is the max over ranks and ``value`` is the whole-job time
per layer-step (max time / (N * K)).
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import statistics
import subprocess
import sys
import tempfile
import time

import numpy as np

HERE = os.path.dirname(os.path.abspath(__file__))
METRIC = "sparse-FFN decode µs/layer + achieved HBM GB/s vs 8 TB/s, speedup over dense"
UNIT = "µs/layer"
NOMINAL_HBM_GBS = 8000.0
FALLBACK_HBM_GBS = 6650.0
D, H = 4096, 11008
N_ROT = 8
N_TOKENS = 64
# Headline path: the one-launch csffn_cats_ffn_forward; the two-call path (csffn_gate_mask +
# csffn_sparse_ffn_forward, same outputs) is reported beside it.
HEADLINE_TWO_CALL = False
# The machine-read figures of the headline kernel's ncu capture (the summary beside it is for people).
PROFILE_JSON = os.path.join(HERE, "profiles", "cats_ring_llama2_7b_b1.json")
TIMED_REPLAYS = 9  # replays of the K-step graph; the headline is their median


def parse_args(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", choices=["csffn", "reference"], default="csffn")
    ap.add_argument("--sparsity", type=float, default=0.5)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-detail", action="store_true", help="skip the 70%/90%/dense detail runs")
    ap.add_argument("--only-dense-verify", action="store_true",
                    help="time only the 70B-shaped 16-token dense verify (for profiling its kernels)")
    ap.add_argument("--rotate", type=int, default=8,
                    help="distinct layer weight sets the steps rotate over (8 keeps every step out of L2; "
                         "1 only for profiler captures, which flush caches themselves)")
    return ap.parse_args(argv)


# ---------------------------------------------------------------------------------- ranks

def dist_env():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return world, rank, local


def init_dist(world, backend):
    import torch.distributed as dist
    if world > 1 and not dist.is_initialized():
        import datetime
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=120))
    return dist


def max_over_ranks(value: float, world: int, device) -> float:
    """Max of a float over ranks (identity for one rank)."""
    if world <= 1:
        return value
    import torch
    import torch.distributed as dist
    t = torch.tensor([value], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def whole_job_us_per_layer(t_max_ms: float, steps: int, world: int) -> float:
    """Whole-job time per layer-step: the slowest rank's time over all ranks' layer-steps."""
    return t_max_ms * 1000.0 / (steps * world)


# ---------------------------------------------------------------------------------- clocks

class ClockSampler:
    """nvidia-smi samples of SM clock and throttle reasons during the measured window."""

    FIELDS = ("index,pci.bus_id,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, bus_id: str):
        self.bus_id = bus_id
        self.proc = None
        self.path = None

    def start(self):
        fd, self.path = tempfile.mkstemp(suffix=".csv")
        os.close(fd)
        try:
            cmd = ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits", "-lms", "100"]
            if self.bus_id:
                cmd += ["-i", self.bus_id]
            self.proc = subprocess.Popen(cmd, stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except OSError:
            self.proc = None
        return self

    def stop(self) -> dict:
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        rows = []
        with open(self.path) as f:
            for line in f:
                parts = [p.strip() for p in line.split(",")]
                if len(parts) >= 10:
                    rows.append(parts)
        os.unlink(self.path)
        sm = [float(r[2]) for r in rows if r[2].replace(".", "").isdigit()]
        mx = [float(r[3]) for r in rows if r[3].replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i in range(4) if r[6 + i].lower() == "active"})
        loaded = [s for s in sm if mx and s > 0.5 * max(mx)] or sm
        return {"sm_mhz": statistics.median(loaded) if loaded else None,
                "sm_max_mhz": max(mx) if mx else None, "reasons": reasons, "samples": len(rows)}


def pci_bus_id(torch, dev: int) -> str:
    try:
        p = torch.cuda.get_device_properties(dev)
        return "%08X:%02X:%02X.0" % (p.pci_domain_id, p.pci_bus_id, p.pci_device_id)
    except Exception:
        return ""


# ---------------------------------------------------------------------------------- peaks

def measured_hbm_gbs():
    path = os.path.join(HERE, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            v = float(json.load(f)["hbm_gbs"])
        return v, "measured"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback"


# Sources of the headline kernel: the profiled traffic is reported only while these are unchanged.
PROFILED_SOURCES = ("ring.cu", "fused_end.cuh", "common.cuh", "tma.cuh", "kernels.h")


def csrc_hash() -> str:
    h = hashlib.sha256()
    d = os.path.join(HERE, "contextual_sparsity_ffn_b200", "csrc")
    for name in PROFILED_SOURCES:
        with open(os.path.join(d, name), "rb") as f:
            h.update(name.encode() + f.read())
    return h.hexdigest()[:16]


def profiled_traffic():
    """DRAM bytes (read + write) per headline-kernel launch from the committed ncu figures, if they
    were taken on this source."""
    try:
        with open(PROFILE_JSON) as f:
            rec = json.load(f)
        traffic = float(rec["traffic_bytes_per_launch"])
        captured = str(rec["csrc_sha256_16"])
    except (OSError, ValueError, KeyError, TypeError):
        return None
    return traffic if captured == csrc_hash() else None


# ---------------------------------------------------------------------------------- csffn arm

def build_workload(torch, cs, synth, sparsities):
    """N_ROT rotation layers on the device, their thresholds per sparsity, and seeded tokens."""
    layers, thresholds = [], {s: [] for s in sparsities}
    for li in range(N_ROT):
        spec, _, xc = synth.llama2_7b_swiglu(li, n_eval=1, n_calib=512)
        layer = cs.FFNLayer.from_spec(spec, "cuda")
        xcal = cs.to_device(xc, "cuda")
        for s in sparsities:
            t = torch.zeros(1, device="cuda")
            cs.calibrate_threshold(layer, xcal, s, 0, t)
            thresholds[s].append(float(t.item()))
        layers.append(layer)
        del spec, xc, xcal
    xs = synth.make_tokens(1, 0, synth.ROLE_EVAL, N_TOKENS, D, "bf16", rms_normalise=True)
    return layers, thresholds, cs.to_device(xs, "cuda")


def run_graph_steps(torch, step_fn, steps, warmup, stream, events_cb=None):
    """Capture `steps` calls of step_fn(k) into one graph; replay warm-up, then time one replay.
    The capture stream first waits for the default stream, where the inputs and workspaces were
    made (a workspace's counters are zeroed there by csffn_workspace_init)."""
    stream.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(stream):
        for k in range(min(warmup, 3)):
            step_fn(k)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=stream, capture_error_mode="relaxed"):
        for k in range(steps):
            step_fn(k)
    return g


def dense_verify_measure(torch, cs, stream, K, W, world, dev):
    """Dense FFN of a 16-token verify chunk on a 70B-shaped layer (d 8192, h 28672, bf16), the
    tensor-core path of csffn_dense_ffn_forward.  Timing only: the weights are drawn on the device
    from a seeded generator (N(0, 0.02^2)); one layer is 1.41 GB, far beyond L2."""
    d, h, B = 8192, 28672, 16
    gen = torch.Generator(device=dev).manual_seed(4)
    w = [(torch.randn(h, d, generator=gen, device=dev) * 0.02).to(torch.bfloat16) for _ in range(3)]
    layer = cs.FFNLayer(w[0], w[1], w[2], cs._abi.ACT_SILU)
    x = (torch.randn(B, d, generator=gen, device=dev)).to(torch.bfloat16)
    o = torch.zeros(B, d, dtype=torch.float32, device=dev)
    ws = cs.new_workspace(layer, B)
    n = max(4, min(K, 20))
    g = run_graph_steps(torch, lambda k: cs.dense_ffn_forward(layer, x, o, ws), n, W, stream)
    for _ in range(2):
        g.replay()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with torch.cuda.stream(stream):
        e0.record()
        g.replay()
        e1.record()
    torch.cuda.synchronize()
    t = max_over_ranks(e0.elapsed_time(e1) * 1e-3, world, dev)
    us_call = t / n * 1e6
    nbytes = 3.0 * 2 * h * d
    flops = 2.0 * B * 3 * h * d
    del g, w, layer, ws
    torch.cuda.empty_cache()
    return {"path": "csffn_dense_ffn_forward, 16 tokens (tensor cores)", "us_per_call": round(us_call, 2),
            "bytes_mb": round(nbytes / 1e6, 1), "achieved_gbs": round(nbytes / (us_call * 1e-6) / 1e9, 1),
            "achieved_tflops": round(flops / (us_call * 1e-6) / 1e12, 1),
            f"frac_of_{measured_hbm_gbs()[1]}_hbm": round(nbytes / (us_call * 1e-6) / 1e9 / measured_hbm_gbs()[0], 4)}


def device_layer(torch, cs, d, h, gen, dev):
    """A bf16 SwiGLU layer drawn on the device from a seeded generator, N(0, 0.02^2) (timing only)."""
    w = [(torch.randn(h, d, generator=gen, device=dev) * 0.02).to(torch.bfloat16) for _ in range(3)]
    return cs.FFNLayer(w[0], w[1], w[2], cs._abi.ACT_SILU)


def time_graph_once(torch, g, stream, warm=2):
    """One timed replay of a captured graph after `warm` untimed ones (ms)."""
    for _ in range(warm):
        g.replay()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with torch.cuda.stream(stream):
        e0.record()
        g.replay()
        e1.record()
    torch.cuda.synchronize()
    return e0.elapsed_time(e1)


def stack_measure(torch, cs, stream, world, dev, n_steps=4):
    """32-layer LLaMA-3-8B-shaped FFN stack (d 4096, h 14336, bf16; 11.3 GB of weights, so every
    step streams from HBM): per layer xn = bf16(RMSNorm(h)) then h += FFN(xn) in place.  Thresholds
    per layer at 50% from 512 calibration vectors carried through the dense stack on the device
    (stack.calibrate_stack).  One step = the 32 layers for B tokens; the residual is reset from the
    same tokens before each step (inside the graph).  The dense stack is timed the same way."""
    from contextual_sparsity_ffn_b200 import stack
    d, h, L = 4096, 14336, 32
    gen = torch.Generator(device=dev).manual_seed(3)
    layers = [device_layer(torch, cs, d, h, gen, dev) for _ in range(L)]
    h_cal = torch.randn(512, d, generator=gen, device=dev)
    ws16 = cs.new_workspace(layers[0], 16)
    ts = stack.calibrate_stack(layers, h_cal, 0.5, ws16)
    h0 = torch.randn(16, d, generator=gen, device=dev)
    res = {"path": "per layer csffn_rmsnorm_bf16 + csffn_cats_ffn_forward (accumulate; batch 1 runs the "
                   "streaming kernel and its finishing kernel, batch 4 and 16 the tensor-core FFN with the "
                   "threshold applied); the dense stack: csffn_rmsnorm_bf16 + csffn_dense_ffn_forward",
           "layers": L, "target_sparsity": 0.5}
    for B in (1, 4, 16):
        sb = stack.stack_buffers(layers[0], B)
        hb = torch.empty(B, d, device=dev)
        counts = []
        hb.copy_(h0[:B])
        stack.sparse_stack(layers, ts, hb, sb, counts=counts)

        def sparse_step(k):
            hb.copy_(h0[:B])
            stack.sparse_stack(layers, ts, hb, sb)

        def dense_step(k):
            hb.copy_(h0[:B])
            stack.dense_stack(layers, hb, sb.xn, ws16)

        g = run_graph_steps(torch, sparse_step, n_steps, 3, stream)
        t_sp = max_over_ranks(time_graph_once(torch, g, stream), world, dev) / n_steps
        del g
        g = run_graph_steps(torch, dense_step, n_steps, 3, stream)
        t_de = max_over_ranks(time_graph_once(torch, g, stream), world, dev) / n_steps
        del g
        assert cs.check_status(sb.buf.ws) == 0
        n_mean = float(np.mean(counts))
        nbytes = 2.0 * h * d + 4.0 * n_mean * d  # per layer: W_gate + the kept W_up / W_down^T rows
        us_l = t_sp * 1e3 / L
        res[f"b{B}"] = {"us_per_step": round(t_sp * 1e3, 1), "us_per_layer": round(us_l, 2),
                        "union_density": round(n_mean / h, 4),
                        "achieved_gbs": round(nbytes / (us_l * 1e-6) / 1e9, 1),
                        "dense_us_per_layer": round(t_de * 1e3 / L, 2),
                        "speedup_vs_dense": round(t_de / t_sp, 3)}
    del layers, ws16
    torch.cuda.empty_cache()
    return res


def sirius_measure(torch, cs, stream, world, dev, rounds=3):
    """Sirius round on LLaMA-3-70B-shaped layers (d 8192, h 28672, bf16, 1.41 GB each): 16 one-token
    sparse drafts (csffn_cats_ffn_forward) then the dense verify of the 16-token chunk
    (csffn_dense_ffn_forward), against 16 dense one-token steps.  Two layers are alternated so no
    step reads weights an earlier one left in L2; times are per layer.  Thresholds from 512
    calibration vectors.  effective_density: weight rows the round reads over those of the 16 dense
    steps (stack.round_effective_density); draft_rel_l2 and top1_agreement compare each draft's output
    with the verify's for the same token (top-1 of a fixed seeded projection to 64 values)."""
    from contextual_sparsity_ffn_b200 import stack
    d, h, T = 8192, 28672, 16
    gen = torch.Generator(device=dev).manual_seed(4)
    layers = [device_layer(torch, cs, d, h, gen, dev) for _ in range(2)]
    xc = torch.randn(512, d, generator=gen, device=dev).to(torch.bfloat16)
    x = torch.randn(T, d, generator=gen, device=dev).to(torch.bfloat16)
    proj = torch.randn(d, 64, generator=gen, device=dev)
    buf = cs.DecodeBuffers.new(layers[0], 1)
    ws_dense = cs.new_workspace(layers[0], T)
    sparse = torch.zeros(T, d, device=dev)
    dense = torch.zeros(T, d, device=dev)
    t_dev = torch.zeros(1, device=dev)
    thresholds = {}
    for s in (0.5, 0.9):
        thresholds[s] = []
        for layer in layers:
            cs.calibrate_threshold(layer, xc, s, cs._abi.CAL_GLOBAL_ABS_ACT, t_dev)
            thresholds[s].append(float(t_dev.item()))
        if not all(math.isfinite(t) for t in thresholds[s]):
            raise RuntimeError(f"calibration gave {thresholds[s]} at s = {s}")

    def dense_tokens(k):
        for layer in layers:
            for j in range(T):
                cs.dense_ffn_forward(layer, x[j:j + 1], dense[j:j + 1], buf.ws)

    g = run_graph_steps(torch, dense_tokens, rounds, 3, stream)
    t_dense = max_over_ranks(time_graph_once(torch, g, stream), world, dev) / (rounds * len(layers))
    del g
    res = {"path": "16 x csffn_cats_ffn_forward (batch 1) + csffn_dense_ffn_forward (batch 16) per layer",
           "dense_16_steps_us_per_layer": round(t_dense * 1e3, 1)}
    for s in (0.5, 0.9):
        ts = thresholds[s]
        rec = []
        stack.sirius_round(layers[0], x, ts[0], sparse, dense, buf, ws_dense, record=rec)
        counts = [len(idx) for idx, _ in rec]
        rel = (torch.linalg.vector_norm(sparse - dense, dim=1) / torch.linalg.vector_norm(dense, dim=1))
        top1 = (torch.argmax(sparse @ proj, dim=1) == torch.argmax(dense @ proj, dim=1)).float()

        def round_step(k):
            for layer, t in zip(layers, ts):
                stack.sirius_round(layer, x, t, sparse, dense, buf, ws_dense)

        g = run_graph_steps(torch, round_step, rounds, 3, stream)
        t_round = max_over_ranks(time_graph_once(torch, g, stream), world, dev) / (rounds * len(layers))
        del g
        assert cs.check_status(buf.ws) == 0 and cs.check_status(ws_dense) == 0
        res[f"s{int(round(s * 100))}"] = {
            "us_per_round_per_layer": round(t_round * 1e3, 1),
            "time_vs_16_dense_steps": round(t_round / t_dense, 4),
            "neuron_density": round(float(np.mean(counts)) / h, 4),
            "effective_density": round(stack.round_effective_density(counts, h), 4),
            "draft_rel_l2_mean": round(float(rel.mean()), 4),
            "top1_agreement": round(float(top1.mean()), 4)}
    del layers, buf, ws_dense
    torch.cuda.empty_cache()
    return res


def svd_reglu_measure(torch, cs, synth, stream, K, world, dev):
    """SVD-predictor ReGLU workload (d 4096, h 11008, bf16, per-neuron thresholds at q = 0.9):
    per step csffn_svd_ffn_forward (y = x U_r, one grid-wide count, then predictor, gate on the
    predicted set, up and down on the active set: one cooperative launch); "parallel" times
    csffn_svd_ffn_forward_parallel (W_up read with
    W_gate on the predicted set); us_two_calls times csffn_predict_lowrank + csffn_cats_ffn_forward
    on the predicted set for the same tokens.  This step reads a few tens of MB, less than L2,
    so L2 is flushed (a 256 MB write) before every step: step time = time of K x (flush + step)
    minus time of K x flush, both as one CUDA graph.  The truncated SVD of W_gate is the offline
    stage (outside the library), done here with torch on the device."""
    spec, x, xc = synth.reglu_sparse(0, d=D, h=H, n_eval=N_TOKENS, n_calib=512)
    layer = cs.FFNLayer.from_spec(spec, "cuda")
    xs = cs.to_device(x, "cuda")
    xcal = cs.to_device(xc, "cuda")
    u, sv, vh = torch.linalg.svd(layer.w_gate.float().T, full_matrices=False)  # W_gate^T = U S V^T
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    n = max(8, min(K, 50))
    out_d = {}
    for r in (256, 1024):
        urt = (u[:, :r] * sv[:r]).T.contiguous().to(torch.bfloat16)
        vr = vh[:r, :].T.contiguous().to(torch.bfloat16)
        tau = torch.zeros(H, device=dev)
        cs.calibrate_threshold(layer, xcal, 0.9, cs._abi.CAL_PER_NEURON_PRED, tau, u_rt=urt, v_r=vr)
        ws = cs.new_workspace(layer, 1, r)
        ci = torch.zeros(H, dtype=torch.int32, device=dev)
        cc = torch.zeros(1, dtype=torch.int32, device=dev)
        idx = torch.zeros(H, dtype=torch.int32, device=dev)
        cnt = torch.zeros(1, dtype=torch.int32, device=dev)
        av = torch.zeros(1, H, device=dev)
        o = torch.zeros(1, D, device=dev)

        def step_two(k):
            x1 = xs[k % N_TOKENS: k % N_TOKENS + 1]
            cs.predict_lowrank(layer, x1, urt, vr, tau, ci, cc, ws)
            cs.cats_ffn_forward(layer, x1, 0.0, idx, cnt, av, o, ws, cand_idx=ci, cand_count=cc)

        def step(k):
            x1 = xs[k % N_TOKENS: k % N_TOKENS + 1]
            cs.svd_ffn_forward(layer, x1, urt, vr, tau, 0.0, idx, cnt, av, o, ws)

        def step_par(k):
            x1 = xs[k % N_TOKENS: k % N_TOKENS + 1]
            cs.svd_ffn_forward(layer, x1, urt, vr, tau, 0.0, idx, cnt, av, o, ws, parallel=True)

        n_p, n_a = [], []
        for k in range(min(n, N_TOKENS)):
            step_two(k)
            n_p.append(int(cc.item()))
            n_a.append(int(cnt.item()))

        def timed(fn):
            def f(k):
                flush.zero_()
                if fn is not None:
                    fn(k)
            g = run_graph_steps(torch, f, n, 3, stream)
            g.replay()
            torch.cuda.synchronize()
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            with torch.cuda.stream(stream):
                e0.record()
                g.replay()
                e1.record()
            torch.cuda.synchronize()
            del g
            return e0.elapsed_time(e1) * 1e3 / n

        t_flush = timed(None)
        us = max_over_ranks(timed(step) - t_flush, world, dev)
        us_par = max_over_ranks(timed(step_par) - t_flush, world, dev)
        us_two = max_over_ranks(timed(step_two) - t_flush, world, dev)
        mp, ma = float(np.mean(n_p)), float(np.mean(n_a))
        # U_r, V_r, the predicted rows' W_gate, the kept rows' W_up and W_down^T (parallel: W_up of
        # every predicted row), flags and index lists
        nbytes = (r * D + H * r) * 2 + mp * D * 2 + 2 * ma * D * 2 + mp * 4 + ma * 8
        nbytes_par = (r * D + H * r) * 2 + 2 * mp * D * 2 + ma * D * 2 + mp * 4 + ma * 8
        out_d[f"r{r}"] = {"us_per_layer": round(us, 2), "predicted_rows": round(mp, 1), "active_rows": round(ma, 1),
                          "bytes_needed_mb": round(nbytes / 1e6, 2),
                          "achieved_gbs": round(nbytes / (us * 1e-6) / 1e9, 1),
                          "launches_per_step": 1,
                          "parallel": {"us_per_layer": round(us_par, 2), "bytes_needed_mb": round(nbytes_par / 1e6, 2),
                                       "achieved_gbs": round(nbytes_par / (us_par * 1e-6) / 1e9, 1)},
                          "us_two_calls": round(us_two, 2)}
        del ws
    del flush, layer
    torch.cuda.empty_cache()
    out_d["path"] = ("csffn_svd_ffn_forward (one cooperative launch); csffn_svd_ffn_forward_parallel beside it; "
                     "L2 flushed before every step")
    return out_d


def csffn_arm(args, world, rank, local):
    import torch
    from contextual_sparsity_ffn_b200 import binding as cs
    from contextual_sparsity_ffn_b200 import synth

    torch.cuda.set_device(local)
    dist = init_dist(world, "nccl")
    dev = torch.device("cuda", local)
    sparsities = [args.sparsity] + ([] if args.no_detail else [s for s in (0.5, 0.7, 0.9) if s != args.sparsity])
    layers, thr, xs = build_workload(torch, cs, synth, sparsities)
    buf = cs.DecodeBuffers.new(layers[0], 1)
    out = torch.zeros(1, D, dtype=torch.float32, device=dev)
    stream = torch.cuda.Stream()
    K, W = args.steps, args.warmup

    def sparse_step(s, events=None, two_call=HEADLINE_TWO_CALL):
        """One decode step on layer k % N_ROT: the one-launch csffn_cats_ffn_forward, or the
        two-call path csffn_gate_mask + csffn_sparse_ffn_forward."""
        def f(k):
            li = k % N_ROT
            x = xs[k % N_TOKENS: k % N_TOKENS + 1]
            if events is not None:
                events[k][0].record()
            if two_call:
                cs.gate_mask(layers[li], x, thr[s][li], buf.idx, buf.count, buf.a_val, buf.ws)
                if events is not None:
                    events[k][1].record()
                cs.sparse_ffn_forward(layers[li], x, buf.idx, buf.count, buf.a_val, out, buf.ws)
            else:
                cs.cats_ffn_forward(layers[li], x, thr[s][li], buf.idx, buf.count, buf.a_val, out, buf.ws)
                if events is not None:
                    events[k][1].record()
        return f

    def dense_step(k):
        li = k % N_ROT
        cs.dense_ffn_forward(layers[li], xs[k % N_TOKENS: k % N_TOKENS + 1], out, buf.ws)

    spread = {}

    def time_graph(g, replays_warm, key=None):
        """Median over TIMED_REPLAYS replays of the K-step graph (ms per replay); each replay is
        bracketed by a barrier and a device synchronise, and timed by events on the capture stream."""
        for _ in range(replays_warm):
            g.replay()
        torch.cuda.synchronize()
        times = []
        for _ in range(TIMED_REPLAYS):
            if world > 1:
                dist.barrier()
            torch.cuda.synchronize()
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            with torch.cuda.stream(stream):
                e0.record()
                g.replay()
                e1.record()
            torch.cuda.synchronize()
            times.append(e0.elapsed_time(e1))
        if world > 1:
            dist.barrier()
        if key is not None:
            spread[key] = {"replays": len(times), "min_ms": round(min(times), 5),
                           "median_ms": round(statistics.median(times), 5), "max_ms": round(max(times), 5)}
        return statistics.median(times)

    # ---- main measurement: K steps at the headline sparsity in one graph, events around the replay.
    # No event nodes inside this graph: they add a gap before every launch (and would break the
    # programmatic dependency between a step's two kernels).  The average step duration is the
    # replay time / K (gaps between steps included).
    g_main = run_graph_steps(torch, sparse_step(args.sparsity), K, W, stream)
    bus = pci_bus_id(torch, local)
    sampler = ClockSampler(bus).start()
    # warm-up: W steps' worth of replays plus a sustained second so clocks settle and are sampled
    warm_replays = max(1, (W + K - 1) // K)
    t_end = time.time() + 1.0
    while time.time() < t_end:
        g_main.replay()
        torch.cuda.synchronize()
    ms = time_graph(g_main, warm_replays, key="headline")
    clocks = sampler.stop()
    ms_max = max_over_ranks(ms, world, dev)
    if HEADLINE_TWO_CALL:
        # the gate kernel's own launches: events around each csffn_gate_mask inside a second graph
        try:
            gate_ev = [(torch.cuda.Event(enable_timing=True, external=True),
                        torch.cuda.Event(enable_timing=True, external=True)) for _ in range(K)]
            g_ev = run_graph_steps(torch, sparse_step(args.sparsity, gate_ev), K, W, stream)
            time_graph(g_ev, warm_replays)
            gate_ms = [a.elapsed_time(b) for a, b in gate_ev]
            del g_ev
        except Exception:
            torch.cuda.synchronize()
            gate_ms = time_step_eager(torch, cs, layers, thr[args.sparsity], xs, buf, out, stream, K)
        kern_avg_us = 1000.0 * float(np.mean(gate_ms))
    else:
        kern_avg_us = 1000.0 * ms / K

    # active rows actually read per step (deterministic; recomputed eagerly)
    counts = []
    for k in range(min(K, N_ROT * N_TOKENS)):
        li = k % N_ROT
        cs.gate_mask(layers[li], xs[k % N_TOKENS: k % N_TOKENS + 1], thr[args.sparsity][li],
                     buf.idx, buf.count, buf.a_val, buf.ws)
        counts.append(int(buf.count.item()))
    n_act = float(np.mean(counts))

    def step_bytes(n_active):
        # all of W_gate + gathered W_up and W_down^T rows + x, out, idx, a_val
        return 2.0 * H * D + 2.0 * 2.0 * n_active * D + 2 * D + 4 * D + 8.0 * n_active

    peak, peak_kind = measured_hbm_gbs()
    us = whole_job_us_per_layer(ms_max, K, world)
    us_gpu = ms_max * 1000.0 / K  # one GPU's time per layer-step
    gbs = step_bytes(n_act) / (us_gpu * 1e-6) / 1e9  # per GPU
    if HEADLINE_TWO_CALL:
        # dominant kernel: the gate (reads all of W_gate); events bracket csffn_gate_mask
        kern_name = "gate_stream_kernel (csffn_gate_mask)"
        kern_bytes = 2.0 * H * D + 2 * D + 8.0 * n_act
    else:
        kern_name = "cats_ring_kernel + ring_finish_kernel (csffn_cats_ffn_forward)"
        kern_bytes = step_bytes(n_act)  # the step's two launches, taken together
    kern_gbs = kern_bytes / (kern_avg_us * 1e-6) / 1e9

    detail = {}
    if not args.no_detail:
        other = not HEADLINE_TWO_CALL
        g = run_graph_steps(torch, sparse_step(args.sparsity, two_call=other), K, W, stream)
        t2 = max_over_ranks(time_graph(g, warm_replays), world, dev)
        u2 = whole_job_us_per_layer(t2, K, world)
        detail[f"{'two_call' if other else 'one_launch'}_{int(round(args.sparsity * 100))}"] = {
            "path": "csffn_gate_mask + csffn_sparse_ffn_forward (3 kernels)" if other
                    else "csffn_cats_ffn_forward (2 kernels)", "us_per_layer": round(u2, 3),
            "achieved_gbs": round(step_bytes(n_act) / (u2 * 1e-6) / 1e9, 1)}
        del g
        for s in sparsities[1:]:
            g = run_graph_steps(torch, sparse_step(s), K, W, stream)
            t = time_graph(g, warm_replays)
            t = max_over_ranks(t, world, dev)
            cnt = []
            for k in range(min(K, N_ROT * N_TOKENS)):
                li = k % N_ROT
                cs.gate_mask(layers[li], xs[k % N_TOKENS: k % N_TOKENS + 1], thr[s][li], buf.idx, buf.count,
                             buf.a_val, buf.ws)
                cnt.append(int(buf.count.item()))
            u = whole_job_us_per_layer(t, K, world)
            detail[f"cats_{int(round(s * 100))}"] = {
                "us_per_layer": round(u, 3), "active_rows": round(float(np.mean(cnt)), 1),
                "bytes_needed_mb": round(step_bytes(np.mean(cnt)) / 1e6, 2),
                "achieved_gbs": round(step_bytes(np.mean(cnt)) / (u * 1e-6) / 1e9, 1),
                "frac_of_8tbs": round(step_bytes(np.mean(cnt)) / (u * 1e-6) / 1e9 / NOMINAL_HBM_GBS, 4)}
            del g
        g = run_graph_steps(torch, dense_step, K, W, stream)
        t = max_over_ranks(time_graph(g, warm_replays), world, dev)
        u = whole_job_us_per_layer(t, K, world)
        dense_bytes = 3.0 * 2 * H * D
        detail["dense"] = {"us_per_layer": round(u, 3), "bytes_needed_mb": round(dense_bytes / 1e6, 2),
                           "achieved_gbs": round(dense_bytes / (u * 1e-6) / 1e9, 1),
                           "frac_of_8tbs": round(dense_bytes / (u * 1e-6) / 1e9 / NOMINAL_HBM_GBS, 4)}
        detail["speedup_vs_dense"] = round(u / us, 3)
        for key in list(detail):
            if key.startswith("cats_"):
                detail[key]["speedup_vs_dense"] = round(u / detail[key]["us_per_layer"], 3)
        del g
        detail["dense_verify_70b_b16"] = dense_verify_measure(torch, cs, stream, K, W, world, dev)
        detail["svd_reglu_q90"] = svd_reglu_measure(torch, cs, synth, stream, K, world, dev)
        detail["stack_llama3_8b_32_layers"] = stack_measure(torch, cs, stream, world, dev)
        detail["sirius_round_70b"] = sirius_measure(torch, cs, stream, world, dev)
    del g_main

    # ---- end to end through the public API: pinned host x in, host out back, every step
    e2e = e2e_measure(torch, cs, layers, thr[args.sparsity], xs, buf, stream, K, W, world, dev)

    result = {
        "metric": METRIC, "value": round(us, 3), "unit": UNIT, "n_gpus": world, "steps": K, "warmup": W,
        "ms_per_step": round(ms_max / K, 6), "higher_is_better": False, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16", "data": "synthetic (seeded N(0,0.02^2) weights, unit-RMS tokens)",
        "config": {"workload": "llama2-7b-shaped SwiGLU FFN layer, batch-1 CATS decode",
                   "d": D, "h": H, "batch": 1, "target_sparsity": args.sparsity,
                   "calibration": "csffn_calibrate_threshold, 512 vectors per layer",
                   "parallelism": f"replicas x{world}" if world > 1 else "single GPU",
                   "l2": f"inputs larger than L2: steps rotate over {N_ROT} layer weight sets "
                         f"({N_ROT * 3 * 2 * H * D / 1e9:.2f} GB)",
                   "timing": f"K steps in one CUDA graph, CUDA events on the capture stream, median of "
                             f"{TIMED_REPLAYS} replays, max over ranks"},
        "tokens_per_s": round(world * K / (ms_max * 1e-3), 1),
        "active_rows": round(n_act, 1),
        "bytes_needed_mb": round(step_bytes(n_act) / 1e6, 2),
        "achieved_gbs": round(gbs, 1),
        "frac_of_8tbs": round(gbs / NOMINAL_HBM_GBS, 4),
        f"frac_of_{peak_kind}_hbm": round(gbs / peak, 4),
        "roofline": {"bound": "hbm", "kernel": kern_name,
                     "achieved": round(kern_gbs, 1), "peak": peak, "unit": "GB/s",
                     "peak_source": f"{peak_kind} copy bandwidth", "frac": round(kern_gbs / peak, 4),
                     "frac_of_8tbs": round(kern_gbs / NOMINAL_HBM_GBS, 4),
                     "traffic": profiled_traffic(), "algorithmic_bytes_per_launch": round(kern_bytes),
                     "avg_launch_us": round(kern_avg_us, 3),
                     "timing": ("events around each csffn_gate_mask launch inside a graph" if HEADLINE_TWO_CALL else
                                "events around each replay of the K-step graph; per step (its two launches and the gap "
                                "between them) = median replay / K"),
                     "replays": spread.get("headline")},
        "e2e": e2e,
        "gpu_launches": (3 if HEADLINE_TWO_CALL else 2) * K,
        "clocks": clocks,
    }
    if detail:
        result["detail"] = detail
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        result["cpu_baseline"] = cpu_baseline(args.sparsity)
    return result, rank


def time_step_eager(torch, cs, layers, thr, xs, buf, out_t, stream, K):
    out = []
    with torch.cuda.stream(stream):
        for k in range(K):
            li = k % N_ROT
            x = xs[k % N_TOKENS: k % N_TOKENS + 1]
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record()
            if HEADLINE_TWO_CALL:
                cs.gate_mask(layers[li], x, thr[li], buf.idx, buf.count, buf.a_val, buf.ws)
            else:
                cs.cats_ffn_forward(layers[li], x, thr[li], buf.idx, buf.count, buf.a_val, out_t, buf.ws)
            b.record()
            if HEADLINE_TWO_CALL:
                cs.sparse_ffn_forward(layers[li], x, buf.idx, buf.count, buf.a_val, out_t, buf.ws)
            out.append((a, b))
    torch.cuda.synchronize()
    return [a.elapsed_time(b) for a, b in out]


def e2e_measure(torch, cs, layers, thr, xs, buf, stream, K, W, world, dev):
    """Same step through the public C-ABI call that takes host buffers (csffn_cats_ffn_forward_host):
    every step takes its token from pinned host memory and puts its output into pinned host memory
    inside the timed region (the step's kernels read x and write out over the host link: a staging
    kernel copies x into the workspace once); the host waits for all K results at the end."""
    host_x = xs.cpu().pin_memory()
    host_out = torch.empty(K, D, dtype=torch.float32).pin_memory()

    def step(k):
        li = k % N_ROT
        cs.cats_ffn_forward_host(layers[li], host_x[k % N_TOKENS: k % N_TOKENS + 1], thr[li], buf.idx, buf.count,
                                 buf.a_val, host_out[k % K: k % K + 1], buf.ws)

    with torch.cuda.stream(stream):
        for k in range(W):
            step(k)
    torch.cuda.synchronize()
    if world > 1:
        import torch.distributed as dist
        dist.barrier()
    t0 = time.perf_counter()
    with torch.cuda.stream(stream):
        for k in range(K):
            step(k)
    torch.cuda.synchronize()
    wall_ms = (time.perf_counter() - t0) * 1e3
    wall_ms = max_over_ranks(wall_ms, world, dev)
    return {"value": round(whole_job_us_per_layer(wall_ms, K, world), 3), "unit": UNIT,
            "h2d_bytes_per_step": 2 * D, "d2h_bytes_per_step": 4 * D,
            "how": "csffn_cats_ffn_forward_host, one C-ABI call per step on pinned host buffers (a "
                   "staging kernel reads x over the host link into the workspace, the step writes out "
                   "into the mapped host buffer); host wall clock around K steps"}


# ---------------------------------------------------------------------------------- oracle legs

def cpu_threads() -> int:
    try:
        from threadpoolctl import threadpool_info
        n = [d.get("num_threads", 1) for d in threadpool_info()]
        return int(max(n)) if n else 1
    except Exception:
        return os.cpu_count() or 1


def cpu_baseline(s: float, budget_s: float = 10.0) -> dict:
    """The CPU oracle as it stands on this host: full 7B-shaped CATS layer calls until ~budget_s."""
    import oracle
    from contextual_sparsity_ffn_b200 import synth

    spec, x, xc = synth.llama2_7b_swiglu(0, n_eval=4, n_calib=512)
    t = oracle.calibrate_global(xc, spec, s)
    times = []
    t_start = time.perf_counter()
    while len(times) < 3 or (time.perf_counter() - t_start < budget_s and len(times) < 64):
        t0 = time.perf_counter()
        oracle.cats_ffn(x[len(times) % 4], spec, t)
        times.append(time.perf_counter() - t0)
    us = 1e6 * statistics.median(times)
    return {"value": round(us, 1), "unit": UNIT, "cores": cpu_threads(), "kind": "oracle",
            "sample": f"{len(times)} full-layer oracle calls (fp64 numpy, d={D}, h={H}, batch 1), median"}


def reference_arm(args, world, rank):
    """The oracle timed on the host cores for the same workload, metric and unit (rank 0 only)."""
    if rank != 0:
        return None, rank
    import oracle
    from contextual_sparsity_ffn_b200 import synth

    spec, x, xc = synth.llama2_7b_swiglu(0, n_eval=4, n_calib=512)
    t = oracle.calibrate_global(xc, spec, args.sparsity)
    # per-step sample: the first h_s neurons of the layer, sized so K + W steps fit ~120 s
    t0 = time.perf_counter()
    oracle.cats_ffn(x[0], spec, t)
    full_s = time.perf_counter() - t0
    budget = 120.0 / max(1, args.steps + args.warmup)
    frac = min(1.0, budget / full_s)
    h_s = max(64, int(H * frac))
    sub = synth.LayerSpec(d=D, h=h_s, dtype=spec.dtype, act=spec.act, w_gate=spec.w_gate[:h_s],
                          w_up=spec.w_up[:h_s], w_down_t=spec.w_down_t[:h_s])
    for k in range(args.warmup):
        oracle.cats_ffn(x[k % 4], sub, t)
    times = []
    for k in range(args.steps):
        t0 = time.perf_counter()
        oracle.cats_ffn(x[k % 4], sub, t)
        times.append(time.perf_counter() - t0)
    total = sum(times)
    us = 1e6 * total / args.steps * (H / h_s)
    sample = (f"each step: oracle CATS FFN over the first {h_s} of {H} neurons (d={D}, batch 1), "
              f"time scaled by {H / h_s:.3f} to a full layer")
    res = {"metric": METRIC, "value": round(us, 1), "unit": UNIT, "n_gpus": world, "steps": args.steps,
           "warmup": args.warmup, "ms_per_step": round(1e3 * total / args.steps, 3), "higher_is_better": False,
           "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
           "config": {"workload": "llama2-7b-shaped SwiGLU FFN layer, batch-1 CATS decode", "d": D, "h": H,
                      "batch": 1, "target_sparsity": args.sparsity},
           "impl": "reference",
           "cpu_baseline": {"value": round(us, 1), "unit": UNIT, "cores": cpu_threads(), "kind": "oracle",
                            "sample": sample},
           "e2e": {"value": round(us, 1), "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    return res, rank


def main(argv=None) -> int:
    global N_ROT
    args = parse_args(argv)
    N_ROT = max(1, args.rotate)
    world, rank, local = dist_env()
    if args.impl == "reference":
        res, rank = reference_arm(args, world, rank)
    elif args.only_dense_verify:
        import torch
        from contextual_sparsity_ffn_b200 import binding as cs
        torch.cuda.set_device(local)
        dev = torch.device("cuda", local)
        res = dense_verify_measure(torch, cs, torch.cuda.Stream(), args.steps, args.warmup, 1, dev)
    else:
        res, rank = csffn_arm(args, world, rank, local)
    if rank == 0 and res is not None:
        print(json.dumps(res), flush=True)
    if world > 1 and args.impl != "reference":
        import torch.distributed as dist
        if dist.is_initialized():
            dist.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
