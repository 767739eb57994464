"""Host logic of the tensor-parallel FFN (no GPU): the row split, the exchange over two gloo ranks
(all-reduce of the partial outputs, all-gather of the calibration activations), and the
decomposition itself against the oracle: the CATS FFN of a layer is the sum of the CATS FFNs of its
row blocks under the same threshold."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import oracle
from contextual_sparsity_ffn_b200 import synth
from contextual_sparsity_ffn_b200 import tensor_parallel as tp


@pytest.mark.parametrize("h,world", [(11008, 2), (11008, 8), (18944, 4), (777, 3), (16, 2), (14336, 7)])
def test_shard_rows_cover_and_align(h, world):
    spans = [tp.shard_rows(h, world, r) for r in range(world)]
    assert spans[0][0] == 0 and spans[-1][1] == h
    for (a0, a1), (b0, b1) in zip(spans, spans[1:]):
        assert a1 == b0  # contiguous, no overlap
    assert all(s0 % tp.SHARD_ALIGN == 0 for s0, _ in spans)
    sizes = [s1 - s0 for s0, s1 in spans]
    assert max(sizes) - min(sizes) < 2 * tp.SHARD_ALIGN  # one group, plus a ragged last group
    with pytest.raises(ValueError):
        tp.shard_rows(h, world, world)


def test_shard_rows_too_few_neurons():
    with pytest.raises(ValueError):
        tp.shard_rows(8, 2, 0)


def _spec_rows(spec, h0, h1):
    return synth.LayerSpec(d=spec.d, h=h1 - h0, dtype=spec.dtype, act=spec.act, w_gate=spec.w_gate[h0:h1],
                           w_up=spec.w_up[h0:h1], w_down_t=spec.w_down_t[h0:h1],
                           bias=spec.bias[h0:h1] if spec.bias is not None else None)


@pytest.mark.parametrize("world", [2, 3, 4])
def test_row_blocks_sum_to_the_layer(world):
    """[CATS] abstract: one threshold for the layer.  The row blocks' CATS outputs add up to the
    layer's, their masks are the layer's mask cut into blocks, and the threshold from all blocks'
    pooled activations is the layer's."""
    spec = synth.make_layer(80, 0, 256, 1000, "bf16")
    x = synth.make_tokens(80, 0, synth.ROLE_EVAL, 3, 256, "bf16", rms_normalise=True)
    xc = synth.make_tokens(80, 0, synth.ROLE_CALIB, 64, 256, "bf16", rms_normalise=True)
    t = oracle.calibrate_global(xc, spec, 0.5)
    full_out, full_mask = oracle.cats_ffn(x, spec, t)
    total = np.zeros_like(full_out)
    pooled = []
    for r in range(world):
        h0, h1 = tp.shard_rows(spec.h, world, r)
        part = _spec_rows(spec, h0, h1)
        out_r, mask_r = oracle.cats_ffn(x, part, t)
        assert np.array_equal(mask_r, full_mask[:, h0:h1])
        total += out_r
        pooled.append(np.abs(oracle.gate_activation(xc, part)))
    assert oracle.rel_l2(total, full_out) <= 1e-12
    vals = np.sort(np.concatenate(pooled, axis=1).ravel())
    k = tp._order_statistic_rank(0.5, vals.size)
    assert k == oracle.order_statistic_rank(0.5, vals.size)
    assert vals[k - 1] == t


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    import datetime
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        spec = synth.make_layer(81, 0, 128, 600, "f32")
        x = synth.make_tokens(81, 0, synth.ROLE_EVAL, 2, 128, "f32", rms_normalise=True)
        t = float(np.quantile(np.abs(oracle.gate_activation(x, spec)), 0.6))
        h0, h1 = tp.shard_rows(spec.h, world, rank)
        out_r, _ = oracle.cats_ffn(x, _spec_rows(spec, h0, h1), t)
        out = torch.from_numpy(out_r.astype(np.float32))
        tp.all_reduce_sum(out)
        absr = torch.from_numpy(np.abs(oracle.gate_activation(x, _spec_rows(spec, h0, h1))).astype(np.float32))
        gathered = tp.gather_abs_activations(absr)
        q.put((rank, out.numpy(), gathered.numpy(), (h0, h1)))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world", [2])
def test_exchange_over_gloo(world):
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = [q.get(timeout=120) for _ in range(world)]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    spec = synth.make_layer(81, 0, 128, 600, "f32")
    x = synth.make_tokens(81, 0, synth.ROLE_EVAL, 2, 128, "f32", rms_normalise=True)
    t = float(np.quantile(np.abs(oracle.gate_activation(x, spec)), 0.6))
    full_out, _ = oracle.cats_ffn(x, spec, t)
    full_abs = np.abs(oracle.gate_activation(x, spec)).astype(np.float32)
    for rank, out, gathered, _ in res:
        assert oracle.rel_l2(out, full_out) <= 1e-6  # every rank holds the layer's output
        assert np.array_equal(gathered, full_abs)     # the ranks' activations in neuron order
