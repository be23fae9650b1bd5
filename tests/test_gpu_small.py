"""GPU parity at sizes the oracle finishes in seconds: the tiny fp32 layer,
bf16 layers spanning several tiles with ragged tails, edge cases, and each
entry point of the C ABI on its own. All calls go through libmoge.so."""
import numpy as np
import pytest
import torch

import mixture_grouped_experts_b200 as mg
import oracle
import synth
from gpu_helpers import (MARGIN, TOL, check_counts, check_routing, device_inputs, layer_parity,
                         normwise_err, run_layer, to_host_f64, x_double)

pytestmark = pytest.mark.gpu

# bf16 layers small enough for the oracle on every token, still several tiles:
# I = 320 -> 5 gate/up feature tiles, d = 512 -> 4 down tiles; ~75 rows per
# expert mixes streaming (<= 64 rows) and tensor tiles; ragged K in "odd".
MED = synth.Config("med", T=300, d=512, N=16, M=4, Kp=1, S=2, I=320, dtype="bf16", seed=11)
CASES = {
    "med": MED,
    "odd": MED.replace(name="odd", T=77, d=520, I=328, seed=12),          # d, I not multiples of 64
    "kp2": MED.replace(name="kp2", T=130, Kp=2, seed=13),                 # 2 picks per group
    "m1": MED.replace(name="m1", T=90, M=1, Kp=2, seed=14),               # one group = global top-2
    "t1": MED.replace(name="t1", T=1, seed=15),                           # single token
    "t17": MED.replace(name="t17", T=17, seed=16),                        # ragged router tile
    "s0": MED.replace(name="s0", T=50, S=0, seed=17),                     # no shared expert
    "big": MED.replace(name="big", T=1100, N=8, M=2, S=1, seed=18),       # > 256 rows per expert
    "n256": MED.replace(name="n256", T=70, N=256, M=8, seed=41),          # router in two 128-row halves
    "n160": MED.replace(name="n160", T=45, N=160, M=8, seed=42),          # groups of 20 (no shuffle path)
    "kp2g8": MED.replace(name="kp2g8", T=120, N=32, M=4, Kp=2, seed=43),  # lane-per-group path, 2 picks
}


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    mg.lib()
    yield
    torch.cuda.synchronize()
    mg.check_device_errors()


def test_tiny_fp32_layer_all_tokens():
    cfg = synth.CONFIGS["tiny"]
    inp = synth.layer_inputs(cfg)
    r = layer_parity(cfg, inp)                 # every token
    assert r["err"] <= TOL["f32"]
    assert r["safe"].sum() >= cfg.T - 4


@pytest.mark.parametrize("name", list(CASES))
def test_bf16_layer_all_tokens(name):
    cfg = CASES[name]
    inp = synth.layer_inputs(cfg)
    layer_parity(cfg, inp)


def test_expert_taking_a_whole_group():
    """Router bias makes one expert of every group take all tokens: the other
    experts get zero rows, the chosen ones T rows (several token tiles)."""
    cfg = MED.replace(name="hot", T=600, seed=19)
    inp = synth.layer_inputs(cfg)
    b = np.full(cfg.N, -30.0, np.float32)
    b[1::cfg.N // cfg.M] = 0.0                  # expert 1 of each group
    inp["logit_bias"] = b
    r = layer_parity(cfg, inp, n_sample=40)
    G = cfg.N // cfg.M
    assert np.array_equal(r["counts"], np.where(np.arange(cfg.N) % G == 1, cfg.T, 0))


def test_route_entry_point_bit_exact_dispatch():
    cfg = MED.replace(name="route", T=333, seed=21)
    inp = synth.layer_inputs(cfg)
    x, w = device_inputs(cfg, inp)
    s = mg.shape_of(cfg)
    ws = mg.alloc_workspace(s)
    idx, wt, counts, offsets, ps, pd = mg.moge_route(s, x, w["w_router"], w["logit_bias"], ws)
    torch.cuda.synchronize()
    idx, wt = idx.cpu().numpy(), wt.cpu().numpy().astype(np.float64)
    xd = x_double(inp, cfg)
    p = oracle.router_probs(xd, inp["w_router"], None, cfg.dtype)
    idx_o, _, mg_o = oracle.select_grouped(p, cfg.M, cfg.Kp)
    safe = check_routing(cfg, p, idx_o, mg_o, idx, wt)
    check_counts(cfg, idx_o, idx, counts.cpu().numpy(), offsets.cpu().numpy(), safe)
    # dispatch of the GPU's own picks is bit-exact with the oracle's definition
    c2, o2, ps2, pd2 = oracle.dispatch(idx, cfg.N)
    assert np.array_equal(counts.cpu().numpy(), c2) and np.array_equal(offsets.cpu().numpy(), o2)
    assert np.array_equal(ps.cpu().numpy(), ps2) and np.array_equal(pd.cpu().numpy(), pd2)


def test_permute_entry_point_is_exact_gather():
    cfg = MED.replace(name="perm", T=200, seed=22)
    inp = synth.layer_inputs(cfg)
    x, _ = device_inputs(cfg, inp)
    s = mg.shape_of(cfg)
    rng = np.random.default_rng(0)
    src = rng.integers(0, cfg.T, cfg.T * cfg.K).astype(np.int32)
    xp = mg.moge_permute(s, x, torch.from_numpy(src).cuda())
    torch.cuda.synchronize()
    got = xp.view(torch.int16).cpu().numpy().view(np.uint16)
    assert np.array_equal(got, inp["x"][src])


def test_grouped_ffn_and_shared_ffn_and_combine_entry_points():
    cfg = MED.replace(name="parts", T=160, seed=23)
    inp = synth.layer_inputs(cfg)
    x, w = device_inputs(cfg, inp)
    s = mg.shape_of(cfg)
    ws = mg.alloc_workspace(s)
    idx, wt, counts, offsets, ps, pd = mg.moge_route(s, x, w["w_router"], None, ws)
    xp = mg.moge_permute(s, x, ps)
    yp = mg.moge_grouped_ffn(s, xp, offsets, w["w_gate"], w["w_up"], w["w_down"], ws)
    ysh = mg.moge_shared_ffn(s, x, w["s_gate"], w["s_up"], w["s_down"], ws)
    y = mg.moge_combine(s, yp, wt, pd, y_shared=ysh)
    y_layer = mg.moge_layer_forward(s, x, w, ws)
    torch.cuda.synchronize()
    mg.check_device_errors()
    xd = x_double(inp, cfg)
    ps_h, idx_h = ps.cpu().numpy(), idx.cpu().numpy()
    off_h = offsets.cpu().numpy()
    yp_h, ysh_h = to_host_f64(yp), to_host_f64(ysh)
    rows = np.random.default_rng(1).choice(cfg.T * cfg.K, 24, replace=False)
    for r in rows:
        e = int(np.searchsorted(off_h, r, side="right") - 1)
        ref = oracle.expert_ffn(xd[ps_h[r]], inp["w_gate"][e], inp["w_up"][e], inp["w_down"][e], "bf16")
        assert normwise_err(yp_h[r], ref) <= TOL["bf16"]
    for t in (0, 77, cfg.T - 1):
        ref = sum(oracle.expert_ffn(xd[t], inp["s_gate"][k], inp["s_up"][k], inp["s_down"][k], "bf16")
                  for k in range(cfg.S))
        assert normwise_err(ysh_h[t], ref) <= TOL["bf16"]
    # the layer call equals the composition of the pieces (same kernels)
    assert normwise_err(to_host_f64(y_layer), to_host_f64(y)) <= 4e-3


def test_combine_residual_and_rmsnorm():
    cfg = MED.replace(name="res", T=64, seed=24)
    inp = synth.layer_inputs(cfg)
    x, w = device_inputs(cfg, inp)
    s = mg.shape_of(cfg)
    ws = mg.alloc_workspace(s)
    u = mg.moge_rmsnorm(s, x, 1e-6)
    y0 = mg.moge_layer_forward(s, u, w, ws)
    y1 = mg.moge_layer_forward(s, u, w, ws, residual=x)
    torch.cuda.synchronize()
    xd = x_double(inp, cfg)
    u_ref = oracle.rmsnorm(xd, 1e-6)
    assert normwise_err(to_host_f64(u), u_ref) <= 4e-3
    assert normwise_err(to_host_f64(y1), to_host_f64(y0) + xd) <= 8e-3


def test_repeat_calls_are_bit_identical():
    cfg = MED.replace(name="det", T=256, seed=25)
    inp = synth.layer_inputs(cfg)
    x, w = device_inputs(cfg, inp)
    s = mg.shape_of(cfg)
    ws = mg.alloc_workspace(s)
    a = mg.moge_layer_forward(s, x, w, ws).clone()
    ws.fill_(0xA5)                                   # poisoned workspace: nothing stale is read
    b = mg.moge_layer_forward(s, x, w, ws)
    torch.cuda.synchronize()
    assert torch.equal(a.view(torch.int16), b.view(torch.int16))


def test_empty_batch_is_a_no_op():
    s = mg.shape_of(MED, T=0)
    ws = mg.alloc_workspace(s)
    x = torch.empty((0, MED.d), dtype=torch.bfloat16, device="cuda")
    inp = synth.layer_inputs(MED.replace(T=1))
    _, w = device_inputs(MED.replace(T=1), inp)
    y = mg.moge_layer_forward(s, x, w, ws)
    idx, wt, counts, offsets, ps, pd = mg.moge_route(s, x, w["w_router"], None, ws)
    torch.cuda.synchronize()
    assert y.shape == (0, MED.d) and int(counts.sum()) == 0 and int(offsets.abs().sum()) == 0


def test_host_buffer_entry_point():
    cfg = MED.replace(name="host", T=96, seed=26)
    inp = synth.layer_inputs(cfg)
    x, w = device_inputs(cfg, inp)
    s = mg.shape_of(cfg)
    ws = mg.alloc_workspace(s)
    ref = mg.moge_layer_forward(s, x, w, ws).clone()
    xh = x.cpu().pin_memory()
    yh = torch.empty_like(xh).pin_memory()
    xd, yd = torch.empty_like(x), torch.empty_like(x)
    mg.moge_layer_forward_host(s, xh, w, ws, yh, xd, yd)
    assert torch.equal(yh.view(torch.int16), ref.cpu().view(torch.int16))


@pytest.mark.parametrize("layout", ["gate_first", "up_first", "same_tensor"])
def test_gate_up_weight_placements(layout):
    """The up-projection fetches its gate+up tile in one copy when w_up lies
    wholly after (or before) w_gate, and in two copies when they overlap (here:
    w_up is w_gate itself). All three give the oracle's result."""
    cfg = MED.replace(name="gu_" + layout, T=120, seed=27)
    inp = synth.layer_inputs(cfg)
    if layout == "same_tensor":
        inp["w_up"] = inp["w_gate"]
    x, w = device_inputs(cfg, inp)
    if layout in ("gate_first", "up_first"):
        n = w["w_gate"].numel()
        both = torch.empty(2 * n, dtype=torch.bfloat16, device="cuda")
        first, second = (both[:n], both[n:])
        g, u = (first, second) if layout == "gate_first" else (second, first)
        g.copy_(w["w_gate"].reshape(-1))
        u.copy_(w["w_up"].reshape(-1))
        w["w_gate"], w["w_up"] = g.view_as(w["w_gate"]), u.view_as(w["w_up"])
        assert (w["w_gate"].data_ptr() < w["w_up"].data_ptr()) == (layout == "gate_first")
    s = mg.shape_of(cfg)
    ws = mg.alloc_workspace(s)
    y, idx_g, w_g, counts_g, offsets_g = run_layer(cfg, x, w, ws)
    xd = x_double(inp, cfg)
    p = oracle.router_probs(xd, inp["w_router"], None, cfg.dtype)
    idx_o, _, mg_o = oracle.select_grouped(p, cfg.M, cfg.Kp)
    safe = check_routing(cfg, p, idx_o, mg_o, idx_g, w_g)
    toks = np.nonzero(safe)[0]
    y_ref, _, _, _ = oracle.layer(xd, inp, cfg.M, cfg.Kp, cfg.dtype, tokens=toks)
    assert normwise_err(to_host_f64(y)[toks], y_ref) <= TOL["bf16"]
