"""GPU parity of the W8A8 layer against the oracle. The weights are E4M3 with
one fp32 scale per row. x and h are quantised per token inside the call, and
both operands of every expert GEMM are E4M3 codes on the 8-bit tensor-core MMA.

* Layer: the oracle quantises the same bf16 weights itself and evaluates the
  W8A8 layer in fp64 (x and h quantised per token with the same rule). The
  GPU layer must match under the usual rules: routing bit-exact above the
  1e-4 margin, outputs within 1e-2 normwise. This is checked at sizes that
  span several tiles with ragged K-chunks and token tails, above 8192 routed
  rows too, and at the decode and prefill workloads on sampled tokens.
* The two sides quantise x identically: bf16 inputs, an exact amax, an IEEE
  fp32 division and round-to-nearest-even.
* h is computed in fp32 on the GPU and in fp64 rounded to fp32 in the oracle.
  A code can differ by one step where the two straddle a rounding boundary;
  such flips are rare and small, and the normwise tolerance covers them.
* Determinism: the same call twice gives the same bytes.
* The W8A8 layer stays close to the weights-only 8-bit layer: the only
  difference is the activation rounding.
"""
import numpy as np
import pytest
import torch

import mixture_grouped_experts_b200 as mg
import oracle
import oracle_par
import synth
from gpu_helpers import (TOL, check_counts, check_routing, device_inputs, normwise_err,
                         sample_tokens, to_host_f64, x_double)

pytestmark = pytest.mark.gpu

MED = synth.Config("a8med", T=300, d=512, N=16, M=4, Kp=1, S=2, I=320, dtype="bf16", seed=41)
CASES = {
    "med": MED,
    "odd": MED.replace(name="a8odd", T=77, d=528, I=336, seed=42),    # ragged 128-code K-chunks
    "kp2": MED.replace(name="a8kp2", T=130, Kp=2, seed=43),
    "t17": MED.replace(name="a8t17", T=17, seed=44),                  # streaming tiles only
    "s0": MED.replace(name="a8s0", T=50, S=0, seed=45),               # no shared expert
    "big": MED.replace(name="a8big", T=1100, N=8, M=2, S=1, seed=46),  # > 256 rows per expert
    "i16": MED.replace(name="a8i16", T=96, d=256, I=16, seed=47),     # one partial K-chunk of h
    # above 8192 routed rows (where the bf16 layer takes the CTA-pair kernel)
    "pair": MED.replace(name="a8pair", T=1100, M=8, seed=51),
    "pair_odd": MED.replace(name="a8pairodd", T=1040, M=8, d=528, I=336, seed=52),
}


def _w8a8_parity(cfg, inp, tokens=None):
    x, w = device_inputs(cfg, inp)
    s = mg.shape_of(cfg)
    ws = mg.alloc_w8a8_workspace(s)
    w8 = mg.experts_to_fp8(w)
    q_o = oracle_par.quantize_experts_fp8(inp)
    for k in mg.FP8_KEYS:                       # the oracle quantised the same weights alike
        if inp[k].size:
            assert np.array_equal(w8[k].cpu().numpy(), q_o[k]), k
    y = mg.moge_layer_forward_w8a8(s, x, w, w8, ws)
    torch.cuda.synchronize()
    mg.check_device_errors()
    idx_g, w_g, counts_g, offsets_g = (a.cpu().numpy() for a in mg.moge_workspace_routing(s, ws))
    xd = x_double(inp, cfg)
    p = oracle.router_probs(xd, inp["w_router"], inp["logit_bias"], cfg.dtype)
    idx_o, _, mg_o = oracle.select_grouped(p, cfg.M, cfg.Kp)
    safe = check_routing(cfg, p, idx_o, mg_o, idx_g, w_g.astype(np.float64))
    check_counts(cfg, idx_o, idx_g, counts_g, offsets_g, safe)
    if tokens is None:
        tokens = np.arange(cfg.T)
    tokens = np.array([t for t in tokens if safe[t]], dtype=np.int64)
    y_ref, _, _, _ = oracle_par.layer_w8a8(xd, inp, q_o, cfg.M, cfg.Kp, cfg.dtype, tokens=tokens)
    err = normwise_err(to_host_f64(y)[tokens], y_ref)
    assert err <= TOL["bf16"], (cfg.name, err)
    return dict(err=err, y=y, x=x, w=w, w8=w8, ws=ws, s=s, tokens=tokens, y_ref=y_ref)


@pytest.mark.parametrize("name", list(CASES))
def test_layer_w8a8_matches_oracle(name):
    cfg = CASES[name]
    _w8a8_parity(cfg, synth.layer_inputs(cfg))


def test_layer_w8a8_elementwise_on_a_small_case():
    """Every output element against the oracle, relative to the row's size: a
    flipped h code moves an element by at most a small fraction of its row."""
    cfg = MED.replace(name="a8el", T=40, d=256, I=128, seed=48)
    r = _w8a8_parity(cfg, synth.layer_inputs(cfg))
    got = to_host_f64(r["y"])[r["tokens"]]
    ref = r["y_ref"]
    row = np.abs(ref).max(axis=1, keepdims=True)
    assert np.all(np.abs(got - ref) <= 2e-2 * row)


def test_layer_w8a8_deterministic_and_close_to_weights_only():
    cfg = MED.replace(name="a8det", T=256, seed=49)
    r = _w8a8_parity(cfg, synth.layer_inputs(cfg))
    y2 = mg.moge_layer_forward_w8a8(r["s"], r["x"], r["w"], r["w8"], r["ws"])
    torch.cuda.synchronize()
    assert torch.equal(r["y"], y2)
    yf = mg.moge_layer_forward_fp8(r["s"], r["x"], r["w"], r["w8"], mg.alloc_workspace(r["s"]))
    torch.cuda.synchronize()
    rel = normwise_err(to_host_f64(y2), to_host_f64(yf))
    assert 0 < rel < 0.1, rel


def test_layer_w8a8_residual():
    cfg = MED.replace(name="a8res", T=64, seed=50)
    inp = synth.layer_inputs(cfg)
    r = _w8a8_parity(cfg, inp)
    res = torch.randn((cfg.T, cfg.d), device="cuda").to(torch.bfloat16)
    y2 = mg.moge_layer_forward_w8a8(r["s"], r["x"], r["w"], r["w8"], r["ws"], residual=res)
    torch.cuda.synchronize()
    want = to_host_f64(r["y"]) + to_host_f64(res)
    assert normwise_err(to_host_f64(y2), want) <= TOL["bf16"]


def test_layer_w8a8_decode_workload_sampled():
    cfg = synth.CONFIGS["decode"]
    inp = synth.layer_inputs(cfg)
    r = _w8a8_parity(cfg, inp, tokens=sample_tokens(cfg.T, 8, seed=5))
    del r
    torch.cuda.empty_cache()


def test_layer_w8a8_prefill_workload_sampled():
    """The prefill workload (T = 4096: about 512 rows per routed expert in two
    256-row token tiles, 16 tiles per shared expert, quantisation items over
    ~190 tiles) on sampled tokens."""
    cfg = synth.CONFIGS["prefill"]
    inp = synth.layer_inputs(cfg)
    r = _w8a8_parity(cfg, inp, tokens=sample_tokens(cfg.T, 6, seed=6))
    del r
    torch.cuda.empty_cache()
