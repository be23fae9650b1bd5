"""GPU parity of layers with more than 8192 routed rows (T * M * K'), whose
grouped FFN runs on CTA pairs (2-SM tensor-core MMA, 256 weight rows per
item): feature and output tiles split between the two CTAs with ragged ends
(I and d not multiples of 128 / 256), experts of every size from streaming
tiles (<= 64 rows) to several 256-row token tiles, and a hot expert."""
import numpy as np
import pytest
import torch

import mixture_grouped_experts_b200 as mg
import synth
from gpu_helpers import layer_parity

pytestmark = pytest.mark.gpu

PAIR_ROWS = 8193  # smallest T * M * K' that takes the pair kernel

BASE = synth.Config("pair", T=2048, d=512, N=64, M=8, Kp=1, S=2, I=384, dtype="bf16", seed=91,
                    w_std=0.05)
CASES = {
    # 9000 routed rows: just past the decode-sized kernel's limit
    "t1125": (BASE.replace(name="pair_t1125", T=1125, seed=96), None),
    # I = 384: three feature pairs, the last one half empty; d = 512: two output pairs
    "even": (BASE, None),
    # d = 520, I = 328: a last output pair of 8 rows, a last feature tile of 8
    "odd": (BASE.replace(name="pair_odd", d=520, I=328, N=32, M=4, Kp=2, seed=92), 700),
    # 256 experts of ~64 rows: streaming and tensor tiles side by side
    "n256": (BASE.replace(name="pair_n256", N=256, S=1, seed=93), 700),
    # no shared expert, 2 picks in each of 2 groups, > 1000 rows per expert
    "s0": (BASE.replace(name="pair_s0", T=4096, N=16, M=2, Kp=2, S=0, seed=94), 600),
}


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    mg.lib()
    yield
    torch.cuda.synchronize()
    mg.check_device_errors()


@pytest.mark.parametrize("name", sorted(CASES))
def test_pair_layer(name):
    cfg, n_sample = CASES[name]
    assert cfg.T * cfg.M * cfg.Kp >= PAIR_ROWS
    layer_parity(cfg, synth.layer_inputs(cfg), n_sample=n_sample)


def test_pair_layer_hot_expert():
    """A router bias sends most tokens of every group to its first expert:
    those experts hold ~1500 rows (six 256-row token tiles), the rest few."""
    cfg = BASE.replace(name="pair_hot", seed=95)
    inp = synth.layer_inputs(cfg)
    bias = np.zeros(cfg.N, dtype=np.float32)
    bias[:: cfg.N // cfg.M] = 1.5
    inp["logit_bias"] = bias
    layer_parity(cfg, inp, n_sample=600)


def test_piecewise_entry_points_at_prefill_size():
    """moge_grouped_ffn and moge_shared_ffn called on their own at the prefill
    workload (32768 routed rows, 16384 shared rows: both above 8192, so both
    run on CTA pairs): sampled rows against the oracle's expert FFN, and the
    pieces composed with moge_combine against the layer call."""
    import oracle
    from gpu_helpers import TOL, device_inputs, normwise_err, to_host_f64, x_double
    cfg = synth.CONFIGS["prefill"]
    assert cfg.T * cfg.K >= PAIR_ROWS and cfg.T * cfg.S >= PAIR_ROWS
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
    ps_h, off_h = ps.cpu().numpy(), offsets.cpu().numpy()
    yp_h = to_host_f64(yp)
    # rows of every kind of token tile: first and last rows of the experts with
    # the most and the fewest rows, and random rows
    cnt = np.diff(off_h)
    rows = []
    for e in (int(cnt.argmax()), int(cnt.argmin()), 0, cfg.N - 1):
        rows += [off_h[e], off_h[e] + cnt[e] // 2, off_h[e + 1] - 1]
    rows += np.random.default_rng(3).choice(cfg.T * cfg.K, 20, replace=False).tolist()
    for r in sorted(set(int(v) for v in rows)):
        e = int(np.searchsorted(off_h, r, side="right") - 1)
        ref = oracle.expert_ffn(xd[ps_h[r]], inp["w_gate"][e], inp["w_up"][e], inp["w_down"][e],
                                "bf16")
        assert normwise_err(yp_h[r], ref) <= TOL["bf16"], (r, e)
    ysh_h = to_host_f64(ysh)
    for t in (0, 255, 256, 2047, cfg.T - 1):
        ref = sum(oracle.expert_ffn(xd[t], inp["s_gate"][k], inp["s_up"][k], inp["s_down"][k],
                                    "bf16") for k in range(cfg.S))
        assert normwise_err(ysh_h[t], ref) <= TOL["bf16"], t
    # the layer call equals the composition of the pieces up to rounding: the
    # pieces round the sum of the shared experts to bf16 (y_shared) before the
    # combine, the layer adds each shared row in fp32 -- one bf16 rounding of
    # a fraction of y more, within the bf16 tolerance
    assert normwise_err(to_host_f64(y_layer), to_host_f64(y)) <= TOL["bf16"]
