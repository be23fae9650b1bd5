"""GPU parity of the layer's backward pass (moge_layer_forward_train +
moge_layer_backward through libmoge.so) against the oracle's fp64 backward,
on the same seeded bf16 inputs and upstream gradient.

Tolerance: every gradient tensor within 2e-2 normwise (max|g - g_ref| /
max|g_ref|). The chain stores three bf16 intermediates in series (the scaled
upstream rows or the pre-activations, the SwiGLU gradients, the result), each
rounding within 2^-9 relatively, and the forward's own tolerance is 1e-2; the
aux loss (fp32 sums) within 1e-3 relatively.

The backward holds the routing at the forward's picks. The GPU's picks are
checked first (bit-exact for every token whose oracle margin exceeds 1e-4, a
valid pick within 1e-4 for the rest, the helpers' forward rule), then the
oracle's backward is run at those same picks."""
import numpy as np
import pytest
import torch

import mixture_grouped_experts_b200 as mg
import oracle
import synth
from gpu_helpers import check_routing, oracle_backward_pool, sample_tokens, to_host_f64

pytestmark = pytest.mark.gpu

TOL = 2e-2


def _normwise(a, ref):
    scale = np.abs(ref).max()
    return float(np.abs(a - ref).max() / scale) if scale > 0 else float(np.abs(a).max())


def _run(cfg, alpha):
    inp = synth.layer_inputs(cfg)
    x = oracle.to_double(inp["x"], cfg.dtype)
    s = mg.shape_of(cfg)
    xd = mg.to_device(inp["x"], cfg.dtype)
    w = mg.weights_to_device(inp, cfg.dtype)
    dy_h = synth.upstream_grad(cfg)
    dy = mg.to_device(dy_h, "bf16")
    ws = mg.alloc_train_workspace(s)
    aux = torch.zeros(1, dtype=torch.float32, device="cuda")
    y = mg.moge_layer_forward_train(s, xd, w, ws)
    idx_g, w_g, _, _ = mg.moge_workspace_routing(s, ws)
    idx_g, w_g = idx_g.cpu().numpy(), w_g.cpu().numpy()
    p = oracle.router_probs(x, inp["w_router"], inp.get("logit_bias"), cfg.dtype)
    idx_o, _, mg_o = oracle.select_grouped(p, cfg.M, cfg.Kp)
    check_routing(cfg, p, idx_o, mg_o, idx_g, w_g)
    dx, grads = mg.moge_layer_backward(s, xd, w, dy, ws, alpha=alpha, aux=aux)
    torch.cuda.synchronize()
    mg.check_device_errors()
    ref = oracle.layer_backward(x, inp, cfg.M, cfg.Kp, cfg.dtype, oracle.to_double(dy_h, "bf16"),
                                alpha, idx=idx_g)
    errs = {"dx": _normwise(to_host_f64(dx), ref["dx"])}
    for k, g in grads.items():
        errs[k] = _normwise(to_host_f64(g), ref[k])
    for k, e in errs.items():
        assert e <= TOL, (cfg.name, k, e, errs)
    if alpha:
        assert abs(float(aux.item()) - ref["aux"]) <= 1e-3 * abs(ref["aux"]), (aux.item(), ref["aux"])
    # the training forward gives the same y as the plain forward
    y2 = mg.moge_layer_forward(s, xd, w, mg.alloc_workspace(s))
    assert torch.equal(y, y2)
    return idx_g, grads, errs


CASES = {
    # several M tiles (I = 192, d = 256 / 384), ragged expert row counts, shared experts
    "s2": synth.Config("bw_s2", T=200, d=256, N=16, M=4, Kp=1, S=2, I=192, dtype="bf16", seed=61,
                       w_std=0.05),
    # K' = 2, wider rows: several N tiles of the weight gradients (d = 640 > 256)
    "kp2": synth.Config("bw_kp2", T=150, d=640, N=16, M=4, Kp=2, S=1, I=128, dtype="bf16",
                        seed=62, w_std=0.05),
    # no shared experts, 64 experts in 8 groups, experts of > 256 rows (two token tiles)
    "n64": synth.Config("bw_n64", T=600, d=256, N=64, M=8, Kp=1, S=0, I=128, dtype="bf16",
                        seed=63, w_std=0.05),
    # 16384 routed rows: the training forward runs the grouped FFN on CTA pairs
    # (g and u kept by that kernel); I = 192: a half-empty last feature pair
    "pair": synth.Config("bw_pair", T=2048, d=256, N=64, M=8, Kp=1, S=1, I=192, dtype="bf16",
                         seed=65, w_std=0.05),
    # 12000 routed rows (the training forward on CTA pairs); d = 320: a last
    # 128-row tile of dx / dW_down half empty; ~375 rows per expert end inside
    # a K chunk of the weight gradients (ragged rows zeroed); 2 picks per group
    "pair_ragged": synth.Config("bw_pair_rag", T=1500, d=320, N=32, M=4, Kp=2, S=2, I=192,
                                dtype="bf16", seed=67, w_std=0.05),
}


@pytest.mark.parametrize("name", sorted(CASES))
def test_backward_matches_oracle(name):
    _run(CASES[name], alpha=0.0)


def test_backward_with_balance_loss():
    _run(CASES["s2"].replace(seed=64), alpha=0.3)


def test_unchosen_experts_get_zero_gradient():
    # 24 tokens over 64 experts (3 per group of 8 on average): several experts
    # take no token; their gradients must be exactly zero
    cfg = synth.Config("bw_sparse", T=24, d=256, N=64, M=8, Kp=1, S=1, I=128, dtype="bf16",
                       seed=65, w_std=0.05)
    idx, grads, _ = _run(cfg, alpha=0.1)
    unused = sorted(set(range(cfg.N)) - set(idx.ravel().tolist()))
    assert unused
    for e in unused:
        for k in ("w_gate", "w_up", "w_down"):
            assert not grads[k][e].float().abs().max().item(), (k, e)


def test_backward_full_size_prefill_sampled():
    """The prefill workload (T = 4096, d = 5120, 64 experts in 8 groups,
    K' = 1, 4 shared experts, I = 1344) in the launch configuration the
    benchmark times. The oracle checks what it can compute one piece at a
    time: dx of sampled tokens, and the complete weight gradients of the
    routed expert with the fewest tokens (its gradient is the sum over exactly
    those tokens). The router gradient is checked by a property that holds at
    any size: its rows sum to zero (each token's softmax gradient does), up to
    the bf16 rounding of dl."""
    cfg = synth.CONFIGS["prefill"]
    alpha = 0.01
    inp = synth.layer_inputs(cfg)
    x = oracle.to_double(inp["x"], cfg.dtype)
    s = mg.shape_of(cfg)
    xd = mg.to_device(inp["x"], cfg.dtype)
    w = mg.weights_to_device(inp, cfg.dtype)
    dy_h = synth.upstream_grad(cfg)
    dy = mg.to_device(dy_h, "bf16")
    ws = mg.alloc_train_workspace(s)
    mg.moge_layer_forward_train(s, xd, w, ws)
    idx_g, w_g, _, _ = mg.moge_workspace_routing(s, ws)
    idx_g, w_g = idx_g.cpu().numpy(), w_g.cpu().numpy()
    dx, grads = mg.moge_layer_backward(s, xd, w, dy, ws, alpha=alpha)
    torch.cuda.synchronize()
    mg.check_device_errors()
    p = oracle.router_probs(x, inp["w_router"], None, cfg.dtype)
    idx_o, _, mg_o = oracle.select_grouped(p, cfg.M, cfg.Kp)
    check_routing(cfg, p, idx_o, mg_o, idx_g, w_g)
    dyd = oracle.to_double(dy_h, "bf16")
    toks = sample_tokens(cfg.T, 6)
    ref = oracle.layer_backward(x, inp, cfg.M, cfg.Kp, cfg.dtype, dyd, alpha, idx=idx_g,
                                tokens=toks, weights=False)
    err = _normwise(to_host_f64(dx)[toks], ref["dx"][toks])
    assert err <= TOL, ("dx", err)
    cnt = np.bincount(idx_g.ravel(), minlength=cfg.N)
    e = int(np.argmin(np.where(cnt > 0, cnt, 1 << 30)))
    rows = np.nonzero((idx_g == e).any(1))[0]
    ref_w = oracle.expert_backward(x[rows], dyd[rows], p[rows, e], inp["w_gate"][e],
                                   inp["w_up"][e], inp["w_down"][e], cfg.dtype)
    for k, r in zip(("w_gate", "w_up", "w_down"), ref_w):
        err = _normwise(to_host_f64(grads[k][e]), r)
        assert err <= TOL, (k, e, len(rows), err)
    gr = grads["w_router"].float()
    assert float(gr.sum(0).abs().max() / gr.abs().max()) <= 0.05


def test_backward_full_dims_small_batch_elementwise():
    """The workload's layer dimensions (d = 5120, 64 experts in 8 groups,
    K' = 1, 4 shared experts, I = 1344) on a batch of 128 tokens, small enough
    for the oracle to form complete gradients: dx of every token, the router's
    gradient and every shared expert's three gradients compared element-wise
    (normwise per tensor), and the routed gradients of the experts with the
    most and the fewest tokens."""
    cfg = synth.Config("bw_full_dims", T=128, d=5120, N=64, M=8, Kp=1, S=4, I=1344,
                       dtype="bf16", seed=66)
    alpha = 0.01
    inp = synth.layer_inputs(cfg)
    x = oracle.to_double(inp["x"], cfg.dtype)
    s = mg.shape_of(cfg)
    xd = mg.to_device(inp["x"], cfg.dtype)
    w = mg.weights_to_device(inp, cfg.dtype)
    dy_h = synth.upstream_grad(cfg)
    ws = mg.alloc_train_workspace(s)
    aux = torch.zeros(1, dtype=torch.float32, device="cuda")
    mg.moge_layer_forward_train(s, xd, w, ws)
    idx_g, w_g, _, _ = mg.moge_workspace_routing(s, ws)
    idx_g, w_g = idx_g.cpu().numpy(), w_g.cpu().numpy()
    dx, grads = mg.moge_layer_backward(s, xd, w, mg.to_device(dy_h, "bf16"), ws, alpha=alpha,
                                       aux=aux)
    torch.cuda.synchronize()
    mg.check_device_errors()
    p = oracle.router_probs(x, inp["w_router"], None, cfg.dtype)
    idx_o, _, mg_o = oracle.select_grouped(p, cfg.M, cfg.Kp)
    check_routing(cfg, p, idx_o, mg_o, idx_g, w_g)
    ref = oracle_backward_pool(cfg, alpha, idx_g, np.arange(cfg.T))
    errs = {"dx": _normwise(to_host_f64(dx), ref["dx"])}
    for k in ("w_router", "s_gate", "s_up", "s_down"):
        errs[k] = _normwise(to_host_f64(grads[k]), ref[k])
    dyd = oracle.to_double(dy_h, "bf16")
    cnt = np.bincount(idx_g.ravel(), minlength=cfg.N)
    for e in (int(np.argmax(cnt)), int(np.argmin(np.where(cnt > 0, cnt, 1 << 30)))):
        rows = np.nonzero((idx_g == e).any(1))[0]
        ref_w = oracle.expert_backward(x[rows], dyd[rows], p[rows, e], inp["w_gate"][e],
                                       inp["w_up"][e], inp["w_down"][e], cfg.dtype)
        for k, r in zip(("w_gate", "w_up", "w_down"), ref_w):
            errs["%s[%d]" % (k, e)] = _normwise(to_host_f64(grads[k][e]), r)
    for k, e in errs.items():
        assert e <= TOL, (k, e, errs)
    assert abs(float(aux.item()) - ref["aux"]) <= 1e-3 * abs(ref["aux"]), (aux.item(), ref["aux"])
