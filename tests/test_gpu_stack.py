"""12-layer stack of MoGE blocks with pre-RMSNorm and residual:
x_{l+1} = x_l + MoGE_l(RMSNorm(x_l)), residual stream stored in bf16.

Two checks per layer and one end to end:
  * teacher forcing: the GPU's own layer input bytes (RMSNorm output) are fed
    to the oracle; the GPU layer output (no residual) on sampled tokens must
    match it, routing bit-exact above the margin;
  * end to end: bf16 drift may flip a pick whose margin is small, after which
    the two stacks legitimately differ. So the oracle's scores on the GPU's own
    layer inputs give every token its smallest in-group margin over the 12
    layers; the tokens with the widest margins (all > 5e-4) are carried
    through the oracle's fp64 stack, must keep the GPU's picks at every layer,
    and must match at the end within sqrt(L) * 1e-2: every layer is held to
    1e-2 of its own output (checked above) and the L layers' independent bf16
    rounding errors, plus the bf16 rounding of the residual after each layer,
    add up roughly in quadrature.
"""
import gc

import numpy as np
import pytest
import torch

import mixture_grouped_experts_b200 as mg
import oracle
import synth
from gpu_helpers import MARGIN, TOL, normwise_err, to_host_f64

pytestmark = pytest.mark.gpu


def _free():
    gc.collect()
    torch.cuda.empty_cache()


def test_stack12_teacher_forced_and_end_to_end():
    cfg = synth.CONFIGS["stack12"]
    s = mg.shape_of(cfg)
    ws = mg.alloc_workspace(s)
    x0 = synth.normal(cfg.seed, synth.STREAM_X, cfg.T * cfg.d, cfg.x_std, "bf16").reshape(cfg.T, cfg.d)
    x_dev = mg.to_device(x0, "bf16")
    min_margin = np.full(cfg.T, np.inf)
    idx_all = []
    checked = 0
    for l in range(cfg.layers):                   # pass 1: the GPU stack
        inp = synth.layer_inputs(cfg, layer=l, with_x=False)
        w = mg.weights_to_device(inp, "bf16")
        u = mg.moge_rmsnorm(s, x_dev, 1e-6)
        y_only = mg.moge_layer_forward(s, u, w, ws)
        x_next = mg.moge_layer_forward(s, u, w, ws, residual=x_dev)
        idx_g = mg.moge_workspace_routing(s, ws)[0].cpu().numpy()
        torch.cuda.synchronize()
        mg.check_device_errors()
        idx_all.append(idx_g)
        u_h = to_host_f64(u)
        p = oracle.router_probs(u_h, inp["w_router"], None, "bf16")
        _, _, mgn = oracle.select_grouped(p, cfg.M, cfg.Kp)
        min_margin = np.minimum(min_margin, mgn)
        # teacher forcing on two tokens per layer
        tf = np.array([(37 * l + 11) % cfg.T, (91 * l + 5) % cfg.T])
        y_ref, idx_ref, _, mg_ref = oracle.layer(u_h, inp, cfg.M, cfg.Kp, "bf16", tokens=tf)
        yg = to_host_f64(y_only)[tf]
        for j, t in enumerate(tf):
            if mg_ref[j] > MARGIN:
                assert np.array_equal(idx_ref[j], idx_g[t]), (l, t)
                assert normwise_err(yg[j], y_ref[j]) <= TOL["bf16"], (l, t)
                checked += 1
        x_dev = x_next
        del w, inp, u, y_only
        _free()
    assert checked >= cfg.layers
    cand = np.argsort(-min_margin)[:4]
    assert np.all(min_margin[cand] > 5e-4), min_margin[cand]
    xo = oracle.to_double(x0, "bf16")[cand]
    for l in range(cfg.layers):                   # pass 2: the oracle's fp64 stack
        inp = synth.layer_inputs(cfg, layer=l, with_x=False)
        yo, idx_o, _, _ = oracle.layer(oracle.rmsnorm(xo, 1e-6), inp, cfg.M, cfg.Kp, "bf16")
        assert np.array_equal(idx_o, idx_all[l][cand]), l
        xo = xo + yo
        del inp
    err = normwise_err(to_host_f64(x_dev)[cand], xo)
    assert err <= np.sqrt(cfg.layers) * TOL["bf16"], err
