"""The expert-parallel decomposition run as two and four gloo ranks on the CPU
(no GPU): each rank owns 1/R of the tokens, all-gathers x, takes its share of
the weights with the library's sharding helper (1/R of the expert groups and
of every shared expert's intermediate features), computes its partial of
the layer with the oracle, and the partials are summed across the ranks (the
reduce-scatter's arithmetic); every rank's rows must then equal the oracle's
whole layer. This checks the sharding and the exchange pattern the CUDA path
uses; the per-rank CUDA partial is checked against the same oracle function
on the GPU."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import mixture_grouped_experts_b200 as mg
import oracle
import synth

CFG = synth.Config("ep_dist", T=16, d=32, N=16, M=4, Kp=1, S=2, I=24, dtype="f32", seed=41,
                   w_std=0.2)


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
        inp = synth.layer_inputs(CFG)
        rows = CFG.T // world
        x_local = torch.from_numpy(inp["x"][rank * rows:(rank + 1) * rows].copy())
        gathered = [torch.empty_like(x_local) for _ in range(world)]
        dist.all_gather(gathered, x_local)
        x_all = torch.cat(gathered).numpy()
        w = {k: torch.from_numpy(inp[k]) for k in ("w_router", "w_gate", "w_up", "w_down",
                                                   "s_gate", "s_up", "s_down")}
        shard = mg.ep_shard_weights(w, rank, world)
        part = oracle.layer_ep_partial(
            oracle.to_double(x_all, "f32"), shard["w_router"].numpy(), None,
            rank * (CFG.N // world), [shard[k].numpy() for k in ("w_gate", "w_up", "w_down")],
            [shard[k].numpy() for k in ("s_gate", "s_up", "s_down")], CFG.N, CFG.M, CFG.Kp, "f32")
        total = torch.from_numpy(part)
        dist.all_reduce(total)  # sum over ranks; this rank keeps its own rows
        mine = total[rank * rows:(rank + 1) * rows].numpy()
        ref, _, _, _ = oracle.layer(oracle.to_double(inp["x"], "f32"), inp, CFG.M, CFG.Kp, "f32",
                                    tokens=range(rank * rows, (rank + 1) * rows))
        out[rank] = {
            "err": float(np.abs(mine - ref).max() / np.abs(ref).max()),
            "x_ok": bool(np.array_equal(x_all, inp["x"])),
            "shapes": [tuple(shard[k].shape) for k in ("w_gate", "s_gate", "s_down")],
        }
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world", [2, 4])
def test_gloo_ranks_expert_parallel_layer(world):
    ctx = mp.get_context("spawn")
    mgr = ctx.Manager()
    out = mgr.dict()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, out)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
    for p in procs:
        if p.is_alive():
            p.kill()
    assert all(p.exitcode == 0 for p in procs)
    for r in range(world):
        assert out[r]["x_ok"]
        assert out[r]["err"] <= 1e-12, out[r]
        n_loc, i_loc = CFG.N // world, CFG.I // world
        assert out[r]["shapes"] == [(n_loc, 24, 32), (2, i_loc, 32), (2, 32, i_loc)]
