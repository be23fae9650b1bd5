"""Pins of the oracle's expert-parallel share of the layer (no GPU): over a
partition of the experts by group and of the shared experts' intermediate
features, the ranks' partials add up to the whole layer (bit for bit at one
rank, to fp64 rounding otherwise), and a rank's partial ignores the other
ranks' weights entirely."""
import numpy as np
import pytest

import oracle
import synth

CFG = synth.Config("ep", T=12, d=32, N=16, M=4, Kp=1, S=2, I=24, dtype="f32", seed=31, w_std=0.2)


def _partials(cfg, inp, world, scramble_others=False):
    x = oracle.to_double(inp["x"], cfg.dtype)
    n_loc, i_s = cfg.N // world, cfg.I // world
    parts = []
    for r in range(world):
        e0, i0 = r * n_loc, r * i_s
        routed = [inp[k][e0:e0 + n_loc] for k in ("w_gate", "w_up", "w_down")]
        shared = [inp["s_gate"][:, i0:i0 + i_s], inp["s_up"][:, i0:i0 + i_s],
                  inp["s_down"][:, :, i0:i0 + i_s]]
        parts.append(oracle.layer_ep_partial(x, inp["w_router"], inp.get("logit_bias"), e0, routed,
                                             shared, cfg.N, cfg.M, cfg.Kp, cfg.dtype))
    return x, parts


@pytest.mark.parametrize("world", [1, 2, 4])
def test_partials_add_up_to_the_layer(world):
    inp = synth.layer_inputs(CFG)
    x, parts = _partials(CFG, inp, world)
    y, _, _, _ = oracle.layer(x, inp, CFG.M, CFG.Kp, CFG.dtype)
    total = np.sum(parts, axis=0)
    if world == 1:
        assert np.array_equal(total, y)
    else:
        np.testing.assert_allclose(total, y, rtol=1e-12, atol=1e-12 * np.abs(y).max())


def test_partial_uses_only_its_own_experts():
    # K' = 2 per group and 8 groups over 4 ranks: a rank's partial is unchanged
    # when every weight it does not hold is replaced
    cfg = synth.Config("ep2", T=9, d=16, N=16, M=8, Kp=2, S=1, I=16, dtype="f32", seed=32,
                       w_std=0.2)
    inp = synth.layer_inputs(cfg)
    x, parts = _partials(cfg, inp, 4)
    other = dict(inp)
    for k in ("w_gate", "w_up", "w_down"):
        a = inp[k].copy()
        a[4:] = -a[4:] * 3.0  # experts outside rank 0's [0, 4)
        other[k] = a
    _, parts2 = _partials(cfg, other, 4)
    assert np.array_equal(parts[0], parts2[0])
    assert not np.array_equal(parts[1], parts2[1])
    total = np.sum(parts, axis=0)
    y, _, _, _ = oracle.layer(x, inp, cfg.M, cfg.Kp, cfg.dtype)
    np.testing.assert_allclose(total, y, rtol=1e-12, atol=1e-12 * np.abs(y).max())
