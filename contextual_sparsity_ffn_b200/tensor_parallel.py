"""Tensor-parallel CATS FFN: the neuron dimension h split across the ranks of a process group.

The weights are neuron-major (row i of W_gate, W_up and W_down^T belongs to neuron i), so a rank's
share of a layer is a contiguous block of rows of each matrix: a view, no copy.  Each rank runs the
library's decode step on its rows (gate, threshold, compaction, up and down all local) into an fp32
partial output, and one all-reduce (sum) over the group gives out.  The threshold t is one number
for the whole layer ("CATS: Contextually-Aware Thresholding for Sparsity in Large Language Models",
abstract: one threshold per layer for a target sparsity), so calibration gathers every rank's
|activations| and selects the global order statistic.

One process per GPU; torch.distributed carries the exchange (NCCL on GPUs).  The exchange is one
all-reduce of B x d fp32 values per layer; the active-index lists stay on their ranks (index j of a
rank's list is neuron h0 + j of the layer).
"""
from __future__ import annotations

from dataclasses import dataclass
from typing import Tuple

import torch

from . import _abi
from . import binding as cs


SHARD_ALIGN = 8  # neurons: shard boundaries keep every row pointer and the bias slice 16-byte aligned


def shard_rows(h: int, world: int, rank: int) -> Tuple[int, int]:
    """Neurons [h0, h1) of rank `rank` out of `world`: contiguous blocks of whole groups of
    SHARD_ALIGN neurons (the last block takes the remainder), the group counts differing by at most
    one, the larger shares first."""
    if world < 1 or not 0 <= rank < world:
        raise ValueError("need 0 <= rank < world")
    groups = (h + SHARD_ALIGN - 1) // SHARD_ALIGN
    if groups < world:
        raise ValueError(f"fewer than {world} groups of {SHARD_ALIGN} neurons")
    base, extra = divmod(groups, world)
    g0 = rank * base + min(rank, extra)
    g1 = g0 + base + (1 if rank < extra else 0)
    return g0 * SHARD_ALIGN, min(h, g1 * SHARD_ALIGN)


@dataclass
class ShardedLayer:
    """A rank's rows of a layer (views of the full matrices) and where they sit in it."""

    layer: cs.FFNLayer
    h0: int
    h1: int
    h_full: int

    @classmethod
    def from_full(cls, full: cs.FFNLayer, world: int, rank: int) -> "ShardedLayer":
        h0, h1 = shard_rows(full.h, world, rank)
        bias = full.bias[h0:h1] if full.bias is not None else None
        part = cs.FFNLayer(full.w_gate[h0:h1], full.w_up[h0:h1], full.w_down_t[h0:h1], full.act, bias)
        return cls(part, h0, h1, full.h)


def global_indices(local_idx: torch.Tensor, shard: ShardedLayer) -> torch.Tensor:
    """A rank's active list (local neuron numbers) as neurons of the full layer."""
    return local_idx + shard.h0


def all_reduce_sum(t: torch.Tensor, group=None) -> None:
    """Sum over the group, in place (a no-op without an initialised process group)."""
    import torch.distributed as dist
    if dist.is_available() and dist.is_initialized():
        dist.all_reduce(t, op=dist.ReduceOp.SUM, group=group)


def tp_cats_forward(shard: ShardedLayer, x: torch.Tensor, t: float, out: torch.Tensor, buf: cs.DecodeBuffers,
                    group=None, stream=None) -> int:
    """One decode step of the sharded layer: csffn_cats_ffn_forward on this rank's rows into out
    (fp32 [B, d], overwritten), then the all-reduce that sums the ranks' partial outputs.  Returns
    this rank's number of active neurons (its list is buf.idx[:n], local numbering)."""
    if out.dtype != torch.float32:
        raise ValueError("the partial outputs are summed in fp32: out must be float32")
    cs.cats_ffn_forward(shard.layer, x, t, buf.idx, buf.count, buf.a_val, out, buf.ws, out_mode=_abi.OUT_F32,
                        stream=stream)
    all_reduce_sum(out, group)
    return int(buf.count.item())


def gather_abs_activations(local_abs: torch.Tensor, group=None) -> torch.Tensor:
    """Every rank's |activation| values [N, h_rank] joined along the neurons -> [N, h] (ranks in
    order).  Without a process group, the local values."""
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()):
        return local_abs
    world = dist.get_world_size(group)
    sizes = [torch.zeros(1, dtype=torch.int64, device=local_abs.device) for _ in range(world)]
    dist.all_gather(sizes, torch.tensor([local_abs.shape[1]], dtype=torch.int64, device=local_abs.device), group=group)
    width = int(max(s.item() for s in sizes))
    padded = torch.zeros(local_abs.shape[0], width, dtype=local_abs.dtype, device=local_abs.device)
    padded[:, :local_abs.shape[1]] = local_abs
    parts = [torch.empty_like(padded) for _ in range(world)]
    dist.all_gather(parts, padded, group=group)
    return torch.cat([p[:, :int(s.item())] for p, s in zip(parts, sizes)], dim=1)


def local_abs_activations(shard: ShardedLayer, x_cal: torch.Tensor, chunk: int = 16) -> torch.Tensor:
    """|act(x W_gate^T + beta)| of this rank's neurons for the calibration tokens [N, d] -> fp32
    [N, h_rank], by csffn_gate_mask with a threshold below every |a| (every neuron kept, so a_val
    holds every activation)."""
    n, h = x_cal.shape[0], shard.layer.h
    out = torch.empty(n, h, dtype=torch.float32, device=x_cal.device)
    buf = cs.DecodeBuffers.new(shard.layer, min(chunk, _abi.MAX_BATCH), device=x_cal.device)
    for b0 in range(0, n, chunk):
        xb = x_cal[b0:b0 + chunk]
        cs.gate_mask(shard.layer, xb, -1.0, buf.idx, buf.count, buf.a_val, buf.ws)
        out[b0:b0 + xb.shape[0]] = buf.a_val[:xb.shape[0], :h].abs()
    return out


def tp_calibrate(shard: ShardedLayer, x_cal: torch.Tensor, target_sparsity: float, group=None) -> float:
    """The layer's CATS threshold from every rank's neurons: the ceil(s * N * h)-th smallest |a|
    over the calibration tokens and all h neurons (0 when that rank is 0), the same number
    csffn_calibrate_threshold gives for the whole layer on one GPU.  Selected with
    csffn_kth_smallest on the gathered values."""
    vals = gather_abs_activations(local_abs_activations(shard, x_cal), group).reshape(-1).contiguous()
    k = _order_statistic_rank(target_sparsity, vals.numel())
    if k == 0:
        return 0.0
    t = torch.zeros(1, dtype=torch.float32, device=vals.device)
    cs.kth_smallest(vals, k, t)
    return float(t.item())


def _order_statistic_rank(s: float, m: int) -> int:
    """ceil(s * m) with s taken at float32 precision and the product evaluated exactly, clamped to
    [0, m] (the rank csffn_calibrate_threshold selects)."""
    from fractions import Fraction
    import math
    import numpy as np
    k = math.ceil(Fraction(float(np.float32(s))) * m)
    return min(max(k, 0), m)


def tp_dense_forward(shard: ShardedLayer, x: torch.Tensor, out: torch.Tensor, ws: torch.Tensor,
                     group=None, stream=None) -> None:
    """The dense FFN of the sharded layer (the verify of a Sirius round): this rank's rows, then
    the all-reduce of the fp32 partial outputs."""
    if out.dtype != torch.float32:
        raise ValueError("out must be float32")
    cs.dense_ffn_forward(shard.layer, x, out, ws, out_mode=_abi.OUT_F32, stream=stream)
    all_reduce_sum(out, group)


def shard_bytes(shard: ShardedLayer) -> int:
    """Weight bytes this rank holds for the layer."""
    es = 2 if shard.layer.dtype == torch.bfloat16 else 4
    return 3 * (shard.h1 - shard.h0) * shard.layer.d * es
