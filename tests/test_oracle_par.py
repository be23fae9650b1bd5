"""The threaded oracle wrappers used by the full-size GPU tests give exactly
what the sequential oracle gives (no GPU): same rows, same order, same bits."""
import numpy as np

import oracle
import oracle_par
import synth

CFG = synth.Config("par", T=37, d=64, N=16, M=4, Kp=2, S=2, I=32, dtype="bf16", seed=71)


def _same(a, b):
    return len(a) == len(b) and all(u.dtype == v.dtype and u.shape == v.shape and
                                    np.array_equal(u, v) for u, v in zip(a, b))


def test_threaded_layers_equal_the_oracle():
    inp = synth.layer_inputs(CFG)
    xd = oracle.to_double(inp["x"], CFG.dtype)
    q = oracle.quantize_experts_fp8(inp)
    q2 = oracle_par.quantize_experts_fp8(inp)
    assert sorted(q) == sorted(q2) and _same([q[k] for k in sorted(q)], [q2[k] for k in sorted(q)])
    for toks in (None, [5, 0, 36, 5, 17], [], list(range(3))):
        assert _same(oracle.layer(xd, inp, CFG.M, CFG.Kp, CFG.dtype, tokens=toks),
                     oracle_par.layer(xd, inp, CFG.M, CFG.Kp, CFG.dtype, tokens=toks))
        assert _same(oracle.layer_fp8(xd, inp, q, CFG.M, CFG.Kp, CFG.dtype, tokens=toks),
                     oracle_par.layer_fp8(xd, inp, q, CFG.M, CFG.Kp, CFG.dtype, tokens=toks))
        assert _same(oracle.layer_w8a8(xd, inp, q, CFG.M, CFG.Kp, CFG.dtype, tokens=toks),
                     oracle_par.layer_w8a8(xd, inp, q, CFG.M, CFG.Kp, CFG.dtype, tokens=toks))


def test_threaded_quantiser_without_shared_experts():
    cfg = CFG.replace(name="par0", S=0, seed=72)
    inp = synth.layer_inputs(cfg)
    q, q2 = oracle.quantize_experts_fp8(inp), oracle_par.quantize_experts_fp8(inp)
    assert sorted(q) == sorted(q2) and _same([q[k] for k in sorted(q)], [q2[k] for k in sorted(q)])


def test_threaded_backward_sum_equals_one_oracle_call():
    """The token terms summed part by part equal one call over all tokens, up
    to the order of the sums; each part's aux is the whole batch's."""
    inp = synth.layer_inputs(CFG)
    xd = oracle.to_double(inp["x"], CFG.dtype)
    dy = oracle.to_double(synth.upstream_grad(CFG), CFG.dtype)
    one = oracle.layer_backward(xd, inp, CFG.M, CFG.Kp, CFG.dtype, dy, 0.01, routed_weights=False)
    idx = oracle.route(xd, inp["w_router"], inp["logit_bias"], CFG.dtype, CFG.M, CFG.Kp)[0]
    for parts in (1, 3, 8):
        got = oracle_par.layer_backward_sum(xd, inp, CFG.M, CFG.Kp, CFG.dtype, dy, 0.01, idx,
                                            None, parts)
        assert sorted(got) == sorted(one)
        assert got["aux"] == one["aux"]
        for k in one:
            if k != "aux":
                assert np.allclose(got[k], one[k], rtol=0, atol=1e-12 * np.abs(one[k]).max()), k
