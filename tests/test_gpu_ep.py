"""GPU parity of the expert-parallel path. One GPU cannot host several ranks
whose kernels run together, and this path has none that wait on one another:
every rank's local step (moge_layer_forward_ep_local) is run in turn on the
one GPU with that rank's share of the weights, each rank's fp32 partial is
compared with the oracle's partial for that rank, and the partials' sum,
finished by moge_ep_finish, with the oracle's whole layer. The
torch.distributed driver (all-gather, local step, reduce-scatter over NCCL,
finish) runs at world size 1. Tolerances and the routing-margin rule are
those of the single-GPU layer (1e-2 bf16, 1e-4 fp32; tokens whose oracle
margin is under 1e-4 are left out of the comparison)."""
import os
import socket

import numpy as np
import pytest
import torch

import mixture_grouped_experts_b200 as mg
import oracle
import synth
from gpu_helpers import MARGIN, TOL, normwise_err, sample_tokens, to_host_f64

pytestmark = pytest.mark.gpu


def _oracle_partial(cfg, inp, x, rank, world, tokens):
    n_loc, i_s = cfg.N // world, cfg.I // world
    e0, i0 = rank * n_loc, rank * i_s
    routed = [inp[k][e0:e0 + n_loc] for k in ("w_gate", "w_up", "w_down")]
    shared = [inp["s_gate"][:, i0:i0 + i_s], inp["s_up"][:, i0:i0 + i_s],
              inp["s_down"][:, :, i0:i0 + i_s]]
    return oracle.layer_ep_partial(x, inp["w_router"], inp.get("logit_bias"), e0, routed, shared,
                                   cfg.N, cfg.M, cfg.Kp, cfg.dtype, tokens=tokens)


def _clear_tokens(cfg, inp, x):
    p = oracle.router_probs(x, inp["w_router"], inp.get("logit_bias"), cfg.dtype)
    _, _, mg_o = oracle.select_grouped(p, cfg.M, cfg.Kp)
    return np.nonzero(mg_o > MARGIN)[0]


CASES = {
    "bf16_w8": (synth.Config("ep8", T=128, d=256, N=64, M=8, Kp=1, S=2, I=256, dtype="bf16",
                             seed=71, w_std=0.05), 8),
    "bf16_w4": (synth.Config("ep4", T=96, d=384, N=32, M=8, Kp=1, S=4, I=192, dtype="bf16",
                             seed=72, w_std=0.05), 4),
    "bf16_w2_kp2": (synth.Config("ep2", T=80, d=256, N=16, M=4, Kp=2, S=1, I=128, dtype="bf16",
                                 seed=73, w_std=0.05), 2),
    "f32_w2": (synth.Config("ep_f32", T=64, d=256, N=16, M=4, Kp=1, S=1, I=128, dtype="f32",
                            seed=74), 2),
}


@pytest.mark.parametrize("name", sorted(CASES))
def test_ranks_in_turn_match_the_oracle(name):
    cfg, world = CASES[name]
    inp = synth.layer_inputs(cfg)
    x = oracle.to_double(inp["x"], cfg.dtype)
    s = mg.shape_of(cfg)
    xd = mg.to_device(inp["x"], cfg.dtype)
    w = mg.weights_to_device(inp, cfg.dtype)
    ws = mg.alloc_ep_workspace(s, world)
    toks = _clear_tokens(cfg, inp, x)
    assert len(toks) >= cfg.T // 2
    total = torch.zeros((cfg.T, cfg.d), dtype=torch.float32, device="cuda")
    for r in range(world):
        part = mg.moge_layer_forward_ep_local(s, r, world, xd, mg.ep_shard_weights(w, r, world), ws)
        torch.cuda.synchronize()
        mg.check_device_errors()
        ref = _oracle_partial(cfg, inp, x, r, world, toks)
        err = normwise_err(to_host_f64(part)[toks], ref)
        assert err <= TOL[cfg.dtype], (name, r, err)
        total += part
    y = mg.moge_ep_finish(s, total)
    y_ref, _, _, _ = oracle.layer(x, inp, cfg.M, cfg.Kp, cfg.dtype, tokens=toks)
    err = normwise_err(to_host_f64(y)[toks], y_ref)
    assert err <= TOL[cfg.dtype], (name, "sum", err)
    # against the single-GPU layer on the same inputs (same picks; the routed
    # rows are summed in another order)
    y1 = mg.moge_layer_forward(s, xd, w, mg.alloc_workspace(s))
    assert normwise_err(to_host_f64(y)[toks], to_host_f64(y1)[toks]) <= TOL[cfg.dtype]


def test_finish_adds_the_residual():
    cfg, _ = CASES["bf16_w4"]
    s = mg.shape_of(cfg)
    g = torch.Generator(device="cuda").manual_seed(5)
    y_sum = torch.randn((cfg.T, cfg.d), generator=g, device="cuda")
    res = torch.randn((cfg.T, cfg.d), generator=g, device="cuda").to(torch.bfloat16)
    y = mg.moge_ep_finish(s, y_sum, res)
    want = (y_sum.double() + res.double()).cpu().numpy()
    got = to_host_f64(y)
    assert np.abs(got - want).max() <= 2.0 ** -8 * np.abs(want).max()


def _free_port():
    sk = socket.socket()
    sk.bind(("127.0.0.1", 0))
    port = sk.getsockname()[1]
    sk.close()
    return port


def test_nccl_driver_world_one():
    import torch.distributed as dist
    cfg, _ = CASES["bf16_w8"]
    inp = synth.layer_inputs(cfg)
    s = mg.shape_of(cfg)
    xd = mg.to_device(inp["x"], cfg.dtype)
    w = mg.weights_to_device(inp, cfg.dtype)
    dist.init_process_group("nccl", init_method="tcp://127.0.0.1:%d" % _free_port(), rank=0,
                            world_size=1)
    try:
        ws = mg.alloc_ep_workspace(s, 1)
        y = mg.moge_layer_forward_ep(s, xd, mg.ep_shard_weights(w, 0, 1), ws, chunks=1)
        # the pipelined schedule: 3 uneven token chunks, gathers on a side
        # stream, each chunk's reduce-scatter overlapping the next chunk's GEMMs
        yc = mg.moge_layer_forward_ep(s, xd, mg.ep_shard_weights(w, 0, 1), ws, chunks=3)
        torch.cuda.synchronize()
        mg.check_device_errors()
    finally:
        dist.destroy_process_group()
    y1 = mg.moge_layer_forward(s, xd, w, mg.alloc_workspace(s))
    x = oracle.to_double(inp["x"], cfg.dtype)
    toks = _clear_tokens(cfg, inp, x)
    assert normwise_err(to_host_f64(y)[toks], to_host_f64(y1)[toks]) <= TOL[cfg.dtype]
    y_ref, _, _, _ = oracle.layer(x, inp, cfg.M, cfg.Kp, cfg.dtype, tokens=toks)
    assert normwise_err(to_host_f64(y)[toks], y_ref) <= TOL[cfg.dtype]
    # a token's result does not depend on the chunk it was computed in (up to
    # the router's split of the hidden dimension, which follows the batch size)
    assert normwise_err(to_host_f64(yc)[toks], to_host_f64(y)[toks]) <= 4e-3


def test_full_size_decode_eight_ranks_sampled():
    """The decode workload (T = 456, d = 5120, 64 experts in 8 groups, K' = 1,
    4 shared, I = 1344) split over 8 ranks, one group each and 168 features of
    every shared expert, the ranks run in turn: sampled tokens of the summed
    partials against the oracle's layer, and one rank's partial against the
    oracle's partial for that rank."""
    cfg = synth.CONFIGS["decode"]
    world = 8
    inp = synth.layer_inputs(cfg)
    x = oracle.to_double(inp["x"], cfg.dtype)
    s = mg.shape_of(cfg)
    xd = mg.to_device(inp["x"], cfg.dtype)
    w = mg.weights_to_device(inp, cfg.dtype)
    ws = mg.alloc_ep_workspace(s, world)
    clear = set(_clear_tokens(cfg, inp, x).tolist())
    toks = np.array([t for t in sample_tokens(cfg.T, 12) if t in clear])
    assert len(toks) >= 8
    total = torch.zeros((cfg.T, cfg.d), dtype=torch.float32, device="cuda")
    for r in range(world):
        part = mg.moge_layer_forward_ep_local(s, r, world, xd, mg.ep_shard_weights(w, r, world), ws)
        if r == 3:
            ref = _oracle_partial(cfg, inp, x, r, world, toks)
            torch.cuda.synchronize()
            assert normwise_err(to_host_f64(part)[toks], ref) <= TOL[cfg.dtype]
        total += part
    torch.cuda.synchronize()
    mg.check_device_errors()
    y = mg.moge_ep_finish(s, total)
    y_ref, _, _, _ = oracle.layer(x, inp, cfg.M, cfg.Kp, cfg.dtype, tokens=toks)
    assert normwise_err(to_host_f64(y)[toks], y_ref) <= TOL[cfg.dtype]
