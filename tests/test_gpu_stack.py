"""12-layer stack of MoGE blocks with pre-RMSNorm and residual:
x_{l+1} = x_l + MoGE_l(RMSNorm(x_l)), residual stream stored in bf16.

Two checks per layer and one end to end:
  * teacher forcing: the GPU's own layer input bytes (RMSNorm output) are fed
    to the oracle; the GPU layer output (no residual) on sampled tokens must
    match it, routing bit-exact above the margin;
  * end to end: candidate tokens carried through the oracle's fp64 stack;
    those whose picks agree with the GPU's at every layer (a pick under the
    margin may legitimately flip with bf16 drift) must match at the end.
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


def test_stack12_teacher_forced_and_end_to_end():
    cfg = synth.CONFIGS["stack12"]
    s = mg.shape_of(cfg)
    ws = mg.alloc_workspace(s)
    x0 = synth.normal(cfg.seed, synth.STREAM_X, cfg.T * cfg.d, cfg.x_std, "bf16").reshape(cfg.T, cfg.d)
    x_dev = mg.to_device(x0, "bf16")
    cand = np.array([3, 50, 101, 222, 333, 455])
    xo = oracle.to_double(x0, "bf16")[cand]
    agree = np.ones(len(cand), bool)
    checked = 0
    for l in range(cfg.layers):
        inp = synth.layer_inputs(cfg, layer=l, with_x=False)
        w = mg.weights_to_device(inp, "bf16")
        u = mg.moge_rmsnorm(s, x_dev, 1e-6)
        y_only = mg.moge_layer_forward(s, u, w, ws)
        x_next = mg.moge_layer_forward(s, u, w, ws, residual=x_dev)
        idx_g = mg.moge_workspace_routing(s, ws)[0].cpu().numpy()
        torch.cuda.synchronize()
        mg.check_device_errors()
        # teacher forcing on two tokens per layer
        u_h = to_host_f64(u)
        tf = np.array([(37 * l + 11) % cfg.T, (91 * l + 5) % cfg.T])
        y_ref, idx_ref, _, mg_ref = oracle.layer(u_h, inp, cfg.M, cfg.Kp, "bf16", tokens=tf)
        yg = to_host_f64(y_only)[tf]
        for j, t in enumerate(tf):
            if mg_ref[j] > MARGIN:
                assert np.array_equal(idx_ref[j], idx_g[t]), (l, t)
                assert normwise_err(yg[j], y_ref[j]) <= TOL["bf16"], (l, t)
                checked += 1
        # the oracle's own fp64 stack for the candidates
        uo = oracle.rmsnorm(xo, 1e-6)
        yo, idx_o, _, _ = oracle.layer(uo, inp, cfg.M, cfg.Kp, "bf16")
        agree &= (idx_o == idx_g[cand]).all(1)
        xo = xo + yo
        x_dev = x_next
        del w, inp, u, y_only
        gc.collect()
        torch.cuda.empty_cache()
    assert checked >= cfg.layers
    assert agree.sum() >= 2, agree
    xg = to_host_f64(x_dev)[cand[agree]]
    err = normwise_err(xg, xo[agree])
    assert err <= TOL["bf16"], err
