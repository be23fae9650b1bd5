"""The data-parallel (N > 1) path of the benchmark, run as two and four gloo
ranks on the CPU: every rank owns a different token batch and the same weights, the
step time is the maximum over ranks, and the job throughput counts every
rank's tokens. No GPU and no collective on the data path."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import bench
import synth

TINY = synth.CONFIGS["tiny"]


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, world, port, out):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        inp = bench.rank_inputs(TINY, rank)
        local_ms = 1.0 + 0.5 * rank                  # later ranks slower
        ms = bench.max_over_ranks(local_ms, True)
        xs = [torch.zeros(TINY.T * TINY.d, dtype=torch.float32) for _ in range(world)]
        dist.all_gather(xs, torch.from_numpy(inp["x"].ravel().copy()))
        ws = [torch.zeros(inp["w_gate"].size, dtype=torch.float32) for _ in range(world)]
        dist.all_gather(ws, torch.from_numpy(inp["w_gate"].ravel().copy()))
        out[rank] = {
            "ms": ms,
            "value": bench.job_throughput(TINY.T, world, ms),
            "x_distinct": all(not torch.equal(xs[i], xs[j])
                              for i in range(world) for j in range(i + 1, world)),
            "w_same": all(torch.equal(ws[0], w) for w in ws[1:]),
        }
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world", [2, 4])
def test_gloo_ranks_weak_scaling_aggregation(world):
    ctx = mp.get_context("spawn")
    mgr = ctx.Manager()
    out = mgr.dict()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, out)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    for r in range(world):
        o = out[r]
        slowest = 1.0 + 0.5 * (world - 1)
        assert o["ms"] == slowest                   # max over ranks, seen by every rank
        assert o["value"] == pytest.approx(world * TINY.T / (slowest * 1e-3))
        assert o["x_distinct"] and o["w_same"]      # own batch, replicated weights


def test_single_process_is_identity():
    assert bench.max_over_ranks(3.25, False) == 3.25
    assert bench.job_throughput(456, 1, 0.5) == pytest.approx(912000.0)
    a = bench.rank_inputs(TINY, 0, with_weights=False)["x"]
    b = bench.rank_inputs(TINY, 1, with_weights=False)["x"]
    assert a.shape == b.shape and not np.array_equal(a, b)
