"""The host-buffer entry points on the GPU: a run of independent batches
through moge_layer_forward_host_stream (copies overlapped with the
neighbouring batches' compute on the library's copy streams) gives every
batch the same output bytes as moge_layer_forward on that batch alone, and
one batch matches the oracle."""
import numpy as np
import pytest
import torch

import mixture_grouped_experts_b200 as mg
import oracle
import synth
from gpu_helpers import MARGIN, TOL, normwise_err, to_host_f64

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("n", [1, 2, 5])
def test_streaming_host_call_equals_device_calls(n):
    cfg = synth.Config("host", T=200, d=512, N=16, M=4, Kp=1, S=2, I=320, dtype="bf16", seed=81,
                       w_std=0.05)
    s = mg.shape_of(cfg)
    inp = synth.layer_inputs(cfg)
    w = mg.weights_to_device(inp, cfg.dtype)
    xs = [synth.layer_inputs(cfg, x_stream_offset=b)["x"] for b in range(n)]
    xh = torch.stack([mg.to_device(a, cfg.dtype).cpu() for a in xs]).pin_memory()
    yh = torch.empty_like(xh).pin_memory()
    xd2 = torch.empty((2, cfg.T, cfg.d), dtype=torch.bfloat16, device="cuda")
    yd2 = torch.empty_like(xd2)
    ws = mg.alloc_workspace(s)
    mg.moge_layer_forward_host_stream(s, xh, w, ws, yh, xd2, yd2)
    mg.check_device_errors()
    for b in range(n):
        y = mg.moge_layer_forward(s, xh[b].cuda(), w, mg.alloc_workspace(s))
        assert torch.equal(y.cpu(), yh[b]), b
    # the last batch against the oracle (tokens above the routing margin)
    x = oracle.to_double(xs[-1], cfg.dtype)
    p = oracle.router_probs(x, inp["w_router"], None, cfg.dtype)
    _, _, mg_o = oracle.select_grouped(p, cfg.M, cfg.Kp)
    toks = np.nonzero(mg_o > MARGIN)[0]
    inp_last = dict(inp)
    inp_last["x"] = xs[-1]
    y_ref, _, _, _ = oracle.layer(x, inp_last, cfg.M, cfg.Kp, cfg.dtype, tokens=toks)
    assert normwise_err(to_host_f64(yh[-1])[toks], y_ref) <= TOL[cfg.dtype]
