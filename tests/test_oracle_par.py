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
