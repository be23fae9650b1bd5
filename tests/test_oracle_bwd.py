"""Pins of the oracle's backward pass (no GPU): central finite differences of
the oracle's own forward layer, coordinate by coordinate, for every input and
weight tensor, with the routing checked to stay put under each perturbation;
the balance loss alone; the dense special case (every expert picked); and the
softmax invariant that the router gradient's rows sum to zero."""
import numpy as np
import pytest

import oracle
import synth

WEIGHTS = ("w_router", "w_gate", "w_up", "w_down", "s_gate", "s_up", "s_down")


def _loss(x, inp, M, Kp, dtype, dy, alpha, f):
    """sum_t dy_t . y_t + alpha sum_i f_i P_i, f fixed (the balance loss's count share)."""
    y, idx, _, _ = oracle.layer(x, inp, M, Kp, dtype)
    p = oracle.router_probs(x, inp["w_router"], inp.get("logit_bias"), dtype)
    return float((dy * y).sum() + alpha * (f * p.mean(0)).sum()), idx


def _count_share(x, inp, M, Kp, dtype, N):
    _, idx, _, _ = oracle.layer(x, inp, M, Kp, dtype)
    return np.bincount(idx.ravel(), minlength=N) / x.shape[0], idx


def _check_fd(cfg, alpha, n_coords=6, h_x=1e-5, h_w=1e-4, tensors=("x",) + WEIGHTS, seed=0):
    inp = synth.layer_inputs(cfg)
    x = oracle.to_double(inp["x"], cfg.dtype)
    rng = np.random.default_rng(seed)
    dy = rng.normal(size=x.shape)
    g = oracle.layer_backward(x, inp, cfg.M, cfg.Kp, cfg.dtype, dy, alpha)
    f, idx0 = _count_share(x, inp, cfg.M, cfg.Kp, cfg.dtype, cfg.N)
    checked = 0
    for name in tensors:
        if name.startswith("s_") and cfg.S == 0:
            continue
        base = x if name == "x" else inp[name]
        ana = g["dx"] if name == "x" else g[name]
        for flat in rng.choice(base.size, size=min(n_coords, base.size), replace=False):
            vals = []
            for sgn in (1.0, -1.0):
                if name == "x":
                    xp = x.copy()
                    xp.flat[flat] += sgn * h_x
                    L, idx = _loss(xp, inp, cfg.M, cfg.Kp, cfg.dtype, dy, alpha, f)
                    vals.append((L, xp.flat[flat]))
                else:
                    w = base.copy()
                    w.flat[flat] = np.float32(w.flat[flat] + sgn * h_w)
                    ip = dict(inp)
                    ip[name] = w
                    L, idx = _loss(x, ip, cfg.M, cfg.Kp, cfg.dtype, dy, alpha, f)
                    vals.append((L, float(w.flat[flat])))
                assert np.array_equal(idx, idx0), "routing moved under the perturbation"
            fd = (vals[0][0] - vals[1][0]) / (vals[0][1] - vals[1][1])
            an = ana.flat[flat]
            assert abs(fd - an) <= 1e-6 * max(1.0, abs(an)), (name, flat, fd, an)
            checked += 1
    return checked


SMALL = synth.Config("fd", T=7, d=24, N=8, M=4, Kp=1, S=2, I=12, dtype="f32", seed=21, w_std=0.3)


def test_fd_every_tensor():
    assert _check_fd(SMALL, alpha=0.0) >= 40


def test_fd_with_balance_loss():
    assert _check_fd(SMALL, alpha=0.37, seed=1) >= 40


def test_fd_balance_loss_alone():
    cfg = SMALL.replace(seed=22)
    inp = synth.layer_inputs(cfg)
    x = oracle.to_double(inp["x"], "f32")
    g = oracle.layer_backward(x, inp, cfg.M, cfg.Kp, "f32", np.zeros_like(x), alpha=1.0)
    # no upstream gradient: only the router and x move, every expert gradient is zero
    for k in ("w_gate", "w_up", "w_down", "s_gate", "s_up", "s_down"):
        assert not g[k].any()
    assert np.abs(g["w_router"]).max() > 0
    f, _ = _count_share(x, inp, cfg.M, cfg.Kp, "f32", cfg.N)
    p = oracle.router_probs(x, inp["w_router"], None, "f32")
    assert g["aux"] == pytest.approx(float((f * p.mean(0)).sum()), rel=1e-12)
    assert _check_fd(cfg, alpha=1.0, tensors=("x", "w_router"), seed=2) >= 12


def test_fd_dense_every_expert_picked():
    # K' = N/M: the picks never change, the layer is sum_e p_e FFN_e(x) + shared
    cfg = synth.Config("dense", T=5, d=16, N=8, M=2, Kp=4, S=1, I=8, dtype="f32", seed=23,
                       w_std=0.3)
    assert _check_fd(cfg, alpha=0.2, seed=3) >= 40


def test_fd_bf16_weights_through_x():
    cfg = SMALL.replace(dtype="bf16", seed=24)
    assert _check_fd(cfg, alpha=0.1, tensors=("x",), n_coords=12, seed=4) == 12


def test_router_gradient_rows_sum_to_zero_and_linearity():
    inp = synth.layer_inputs(SMALL)
    x = oracle.to_double(inp["x"], "f32")
    dy = np.random.default_rng(5).normal(size=x.shape)
    g1 = oracle.layer_backward(x, inp, SMALL.M, SMALL.Kp, "f32", dy, 0.0)
    g2 = oracle.layer_backward(x, inp, SMALL.M, SMALL.Kp, "f32", 2.0 * dy, 0.0)
    assert np.abs(g1["w_router"].sum(0)).max() < 1e-12
    for k in ("dx",) + WEIGHTS:
        np.testing.assert_allclose(g2[k], 2.0 * g1[k], rtol=1e-12, atol=1e-14)


def test_routing_override():
    # held at its own picks the override changes nothing; at another valid pick
    # of a group the gradients move; a pick outside its group is refused
    inp = synth.layer_inputs(SMALL)
    x = oracle.to_double(inp["x"], "f32")
    dy = np.random.default_rng(6).normal(size=x.shape)
    _, idx, _, _ = oracle.layer(x, inp, SMALL.M, SMALL.Kp, "f32")
    a = oracle.layer_backward(x, inp, SMALL.M, SMALL.Kp, "f32", dy, 0.2)
    b = oracle.layer_backward(x, inp, SMALL.M, SMALL.Kp, "f32", dy, 0.2, idx=idx)
    for k in ("dx",) + WEIGHTS:
        assert np.array_equal(a[k], b[k])
    G = SMALL.N // SMALL.M
    other = idx.copy()
    other[0, 0] = (other[0, 0] + 1) % G  # group 0 holds experts 0 .. G-1
    c = oracle.layer_backward(x, inp, SMALL.M, SMALL.Kp, "f32", dy, 0.2, idx=other)
    assert not np.array_equal(a["w_gate"], c["w_gate"])
    bad = idx.copy()
    bad[0, 0] = SMALL.N - 1
    with pytest.raises(ValueError):
        oracle.layer_backward(x, inp, SMALL.M, SMALL.Kp, "f32", dy, 0.2, idx=bad)


def test_token_subset_and_per_expert_gradients():
    # a token subset gives those tokens' dx rows exactly; one expert's weight
    # gradient from only the tokens that chose it is that expert's whole gradient
    cfg = SMALL.replace(T=11, seed=25)
    inp = synth.layer_inputs(cfg)
    x = oracle.to_double(inp["x"], "f32")
    dy = np.random.default_rng(7).normal(size=x.shape)
    full = oracle.layer_backward(x, inp, cfg.M, cfg.Kp, "f32", dy, 0.3)
    sub = [2, 5, 9]
    part = oracle.layer_backward(x, inp, cfg.M, cfg.Kp, "f32", dy, 0.3, tokens=sub)
    assert np.array_equal(part["dx"][sub], full["dx"][sub])
    assert not part["dx"][[0, 1, 3]].any()
    p = oracle.router_probs(x, inp["w_router"], None, "f32")
    idx, _, _ = oracle.select_grouped(p, cfg.M, cfg.Kp)
    for e in range(cfg.N):
        rows = np.nonzero((idx == e).any(1))[0]
        dwg, dwu, dwd = oracle.expert_backward(x[rows], dy[rows], p[rows, e], inp["w_gate"][e],
                                               inp["w_up"][e], inp["w_down"][e], "f32")
        assert np.array_equal(dwg, full["w_gate"][e])
        assert np.array_equal(dwu, full["w_up"][e])
        assert np.array_equal(dwd, full["w_down"][e])
    one = np.ones(cfg.T)
    dsg, dsu, dsd = oracle.expert_backward(x, dy, one, inp["s_gate"][1], inp["s_up"][1],
                                           inp["s_down"][1], "f32")
    assert np.array_equal(dsg, full["s_gate"][1]) and np.array_equal(dsd, full["s_down"][1])


def test_dx_only():
    cfg = SMALL.replace(T=9, seed=26)
    inp = synth.layer_inputs(cfg)
    x = oracle.to_double(inp["x"], "f32")
    dy = np.random.default_rng(8).normal(size=x.shape)
    full = oracle.layer_backward(x, inp, cfg.M, cfg.Kp, "f32", dy, 0.2)
    only = oracle.layer_backward(x, inp, cfg.M, cfg.Kp, "f32", dy, 0.2, weights=False)
    assert set(only) == {"dx", "aux"}
    assert np.array_equal(only["dx"], full["dx"])


def test_backward_without_routed_weight_gradients_changes_nothing_else():
    """routed_weights=False leaves out only the routed experts' gradient arrays:
    dx, the router's and the shared experts' gradients and L_aux are the full
    run's, bit for bit."""
    cfg = synth.Config("bw_sel", T=12, d=48, N=8, M=4, Kp=1, S=2, I=24, dtype="f32", seed=71,
                       w_std=0.3)
    inp = synth.layer_inputs(cfg)
    x = oracle.to_double(inp["x"], cfg.dtype)
    dy = oracle.to_double(synth.upstream_grad(cfg), cfg.dtype)
    full = oracle.layer_backward(x, inp, cfg.M, cfg.Kp, cfg.dtype, dy, 0.2)
    part = oracle.layer_backward(x, inp, cfg.M, cfg.Kp, cfg.dtype, dy, 0.2, routed_weights=False)
    assert "w_gate" not in part and "w_up" not in part and "w_down" not in part
    for k in ("dx", "w_router", "s_gate", "s_up", "s_down"):
        assert np.array_equal(full[k], part[k]), k
    assert full["aux"] == part["aux"]
