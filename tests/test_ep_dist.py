"""The expert-parallel decomposition run as two and four gloo ranks on the CPU
(no GPU): each rank owns 1/R of the tokens, all-gathers x, takes its share of
the weights with the library's sharding helper (1/R of the expert groups and
of every shared expert's intermediate features), computes its partial of
the layer with the oracle, and the partials are summed across the ranks (the
reduce-scatter's arithmetic); every rank's rows must then equal the oracle's
whole layer. This checks the sharding and the exchange pattern the CUDA path
uses; the per-rank CUDA partial is checked against the same oracle function
on the GPU. The pipelined schedule (token chunks, each gathered, computed,
reduced and finished in turn: mixture_grouped_experts_b200.ep_pipeline) runs
here too, with gloo's collectives in place of NCCL's."""
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


def _pipeline_worker(rank, world, port, chunks, out):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        inp = synth.layer_inputs(CFG)
        rows = CFG.T // world
        x_local = torch.from_numpy(inp["x"][rank * rows:(rank + 1) * rows].copy())
        w = {k: torch.from_numpy(inp[k]) for k in ("w_router", "w_gate", "w_up", "w_down",
                                                   "s_gate", "s_up", "s_down")}
        shard = mg.ep_shard_weights(w, rank, world)
        seen = []

        def gather(xc):  # all ranks' rows of this chunk, rank-major
            lst = [torch.empty_like(xc) for _ in range(world)]
            dist.all_gather(lst, xc.contiguous())
            return torch.cat(lst)

        def local(xa):  # this rank's partial of the chunk's tokens
            seen.append(xa.shape[0])
            return torch.from_numpy(oracle.layer_ep_partial(
                oracle.to_double(xa.numpy(), "f32"), shard["w_router"].numpy(), None,
                rank * (CFG.N // world), [shard[k].numpy() for k in ("w_gate", "w_up", "w_down")],
                [shard[k].numpy() for k in ("s_gate", "s_up", "s_down")], CFG.N, CFG.M, CFG.Kp,
                "f32"))

        def reduce(part):  # the reduce-scatter's result: the sum, this rank's rows
            t = part.clone()
            dist.all_reduce(t)
            cr = part.shape[0] // world
            return t[rank * cr:(rank + 1) * cr]

        bounds = mg.ep_chunk_bounds(rows, chunks)
        outs = mg.ep_pipeline(x_local, bounds, gather, local, reduce,
                              lambda a, b, ysum: (a, b, ysum.numpy()))
        mine = np.concatenate([o[2] for o in outs])
        ref, _, _, _ = oracle.layer(oracle.to_double(inp["x"], "f32"), inp, CFG.M, CFG.Kp, "f32",
                                    tokens=range(rank * rows, (rank + 1) * rows))
        out[rank] = {"err": float(np.abs(mine - ref).max() / np.abs(ref).max()),
                     "bounds": bounds, "seen": seen}
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world,chunks", [(2, 3), (4, 3), (2, 1)])
def test_gloo_ranks_pipelined_chunks(world, chunks):
    """Token chunks of uneven size (8 rows in 3 chunks: 3, 3, 2; 4 rows: 2, 1, 1):
    each chunk's gathered batch holds world times its rows, and the rows each
    rank gets back, chunk by chunk, are the oracle's layer for its tokens."""
    ctx = mp.get_context("spawn")
    mgr = ctx.Manager()
    out = mgr.dict()
    port = _free_port()
    procs = [ctx.Process(target=_pipeline_worker, args=(r, world, port, chunks, out))
             for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
    for p in procs:
        if p.is_alive():
            p.kill()
    assert all(p.exitcode == 0 for p in procs)
    rows = CFG.T // world
    want = mg.ep_chunk_bounds(rows, chunks)
    assert want[0][0] == 0 and want[-1][1] == rows and len(want) == min(chunks, rows)
    for r in range(world):
        assert out[r]["bounds"] == want
        assert out[r]["seen"] == [world * (b - a) for a, b in want]
        assert out[r]["err"] <= 1e-12, out[r]


def test_chunk_bounds_partition_every_rank_alike():
    """The chunks cover a rank's rows in order, without gaps or empty chunks,
    their sizes differ by at most one, and more chunks than rows are clipped;
    decode-sized batches stay one chunk."""
    for rows in (0, 1, 2, 7, 8, 100, 457):
        for chunks in (1, 2, 3, 4, 9, 1000):
            b = mg.ep_chunk_bounds(rows, chunks)
            assert len(b) == (max(1, min(chunks, rows)) if rows else 1)
            assert b[0][0] == 0 and b[-1][1] == rows
            assert all(b[j][1] == b[j + 1][0] for j in range(len(b) - 1))
            sizes = [hi - lo for lo, hi in b]
            assert max(sizes) - min(sizes) <= 1
            assert rows == 0 or min(sizes) >= 1
    assert [mg.ep_default_chunks(r) for r in (1, 456, 511, 512, 767, 768, 1024, 4096)] == \
        [1, 1, 1, 2, 2, 3, 4, 4]
