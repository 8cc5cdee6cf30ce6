"""Data-parallel host logic on CPU: token shards and the gradient all-reduce
over a world of two gloo ranks, checked against the full-batch oracle."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import oracle
from activation_sparse_transformer_tma_b200 import dp, synth


@pytest.mark.parametrize("T,world", [(0, 1), (1, 2), (7, 2), (64, 2), (65, 4), (3, 8)])
def test_shards_cover_tokens_once(T, world):
    spans = [dp.shard(T, r, world) for r in range(world)]
    assert spans[0][0] == 0 and spans[-1][1] == T
    for (a0, b0), (a1, b1) in zip(spans, spans[1:]):
        assert b0 == a1
    sizes = [b - a for a, b in spans]
    assert max(sizes) - min(sizes) <= 1


def test_shard_rejects_bad_arguments():
    with pytest.raises(ValueError):
        dp.shard(8, 2, 2)
    with pytest.raises(ValueError):
        dp.shard(8, 0, 0)


def _workload():
    return synth.make_workload(T=48, d=32, F=256, W=128, C=8, C_h=16, dtype=synth.BF16,
                               kind="pareto", lam=2e-5, seed=11, mean_active=20.0)


def _rank(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        w = _workload()
        x, Wg, Wu, Wd, dy = (synth.widen(w[k], synth.BF16) for k in ("x", "Wg_t", "Wu_t", "Wd", "dy"))
        a, b = dp.shard(w["T"], rank, world)
        _, dWg, dWu, dWd = oracle.dense_ffn_backward(x[a:b], Wg, Wu, Wd, dy[a:b], w["lam"])
        buf = dp.GradBuffer(w["F"], w["d"], "cpu", dtype=torch.float64)
        buf.dWg_t.copy_(torch.from_numpy(dWg))
        buf.dWu_t.copy_(torch.from_numpy(dWu))
        buf.dWd.copy_(torch.from_numpy(dWd))
        buf.allreduce()
        out[rank] = buf.flat.numpy().copy()
    finally:
        dist.destroy_process_group()


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def test_gradient_allreduce_equals_full_batch():
    world = 2
    out = mp.Manager().dict()
    mp.spawn(_rank, args=(world, _free_port(), out), nprocs=world, join=True)
    w = _workload()
    x, Wg, Wu, Wd, dy = (synth.widen(w[k], synth.BF16) for k in ("x", "Wg_t", "Wu_t", "Wd", "dy"))
    _, dWg, dWu, dWd = oracle.dense_ffn_backward(x, Wg, Wu, Wd, dy, w["lam"])
    ref = np.stack([dWg, dWu, dWd])
    scale = np.abs(ref).max()
    for r in range(world):
        # the same sum, only grouped by shard: equal up to fp64 rounding
        assert np.max(np.abs(out[r] - ref)) <= 1e-12 * scale
    assert np.array_equal(out[0], out[1])
