"""GPU parity of the 8-bit expert-weight path (weights-only FP8, E4M3 codes
with one fp32 scale per weight row) against the oracle.

  * quantisation: codes and scales bit-exact with the oracle's quantiser
    (byte work; both sides divide in IEEE fp32 and round to nearest even);
  * layer: the oracle quantises the same bf16 weights itself and evaluates
    the layer on the dequantised matrices in fp64; the GPU layer must match
    under the usual rules (routing bit-exact above the 1e-4 margin, outputs
    within 1e-2 normwise) -- at sizes that span several tiles with ragged
    tails, and at the decode workload on sampled tokens;
  * determinism: the same call twice gives the same bytes.
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

MED = synth.Config("f8med", T=300, d=512, N=16, M=4, Kp=1, S=2, I=320, dtype="bf16", seed=31)
CASES = {
    "med": MED,
    "odd": MED.replace(name="f8odd", T=77, d=528, I=336, seed=32),    # d, I not multiples of 64
    "kp2": MED.replace(name="f8kp2", T=130, Kp=2, seed=33),
    "t17": MED.replace(name="f8t17", T=17, seed=34),                  # streaming tiles only
    "s0": MED.replace(name="f8s0", T=50, S=0, seed=35),               # no shared expert
    "big": MED.replace(name="f8big", T=1100, N=8, M=2, S=1, seed=36),  # > 256 rows per expert
}


def _bits(t: torch.Tensor) -> np.ndarray:
    return t.contiguous().view(torch.int16).cpu().numpy().view(np.uint16)


def test_quantize_bit_exact_with_oracle():
    rng = np.random.default_rng(5)
    w = rng.normal(0, 0.02, (3, 40, 264)).astype(np.float32)
    w[0, 3] = 0.0                       # all-zero row
    w[1, 7] *= 1e-5                     # codes in the subnormal range
    w[2, 11, 100] = 5.0                 # an outlier sets the row's scale
    w[2, 12, :] = 448.0 * 2.0 ** -3     # all values on one code
    bits = synth.round_bf16(w)
    q_o, s_o = oracle.quantize_rows_fp8(bits)
    wd = torch.from_numpy(bits.view(np.int16)).cuda().view(torch.bfloat16)
    q_g, s_g = mg.moge_quantize_fp8_rows(wd)
    torch.cuda.synchronize()
    assert np.array_equal(s_g.cpu().numpy().view(np.uint32), s_o.view(np.uint32))
    assert np.array_equal(q_g.cpu().numpy(), q_o)


def _fp8_parity(cfg, inp, tokens=None):
    x, w = device_inputs(cfg, inp)
    s = mg.shape_of(cfg)
    ws = mg.alloc_workspace(s)
    w8 = mg.experts_to_fp8(w)
    q_o = oracle_par.quantize_experts_fp8(inp)
    for k in mg.FP8_KEYS:                       # the oracle quantised the same weights alike
        if inp[k].size:
            assert np.array_equal(w8[k].cpu().numpy(), q_o[k]), k
            assert np.array_equal(w8[k + "_scale"].cpu().numpy().view(np.uint32),
                                  q_o[k + "_scale"].view(np.uint32)), k
    y = mg.moge_layer_forward_fp8(s, x, w, w8, ws)
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
    y_ref, _, _, _ = oracle_par.layer_fp8(xd, inp, q_o, cfg.M, cfg.Kp, cfg.dtype, tokens=tokens)
    err = normwise_err(to_host_f64(y)[tokens], y_ref)
    assert err <= TOL["bf16"], (cfg.name, err)
    return dict(err=err, y=y, x=x, w=w, w8=w8, ws=ws, s=s)


@pytest.mark.parametrize("name", list(CASES))
def test_layer_fp8_matches_oracle(name):
    cfg = CASES[name]
    _fp8_parity(cfg, synth.layer_inputs(cfg))


def test_layer_fp8_deterministic_and_close_to_bf16():
    cfg = MED.replace(name="f8det", T=256, seed=37)
    inp = synth.layer_inputs(cfg)
    r = _fp8_parity(cfg, inp)
    y2 = mg.moge_layer_forward_fp8(r["s"], r["x"], r["w"], r["w8"], r["ws"])
    torch.cuda.synchronize()
    assert torch.equal(r["y"], y2)
    # the 8-bit weights stay close to the bf16 layer (quantisation error only)
    yb = mg.moge_layer_forward(r["s"], r["x"], r["w"], r["ws"])
    torch.cuda.synchronize()
    rel = normwise_err(to_host_f64(y2), to_host_f64(yb))
    assert rel < 0.1, rel


def test_layer_fp8_decode_workload_sampled():
    cfg = synth.CONFIGS["decode"]
    inp = synth.layer_inputs(cfg)
    r = _fp8_parity(cfg, inp, tokens=sample_tokens(cfg.T, 8, seed=3))
    del r
    torch.cuda.empty_cache()
