"""Pins of the oracle's 8-bit expert-weight functions (CPU only).

The E4M3 codec is pinned to the format's published constants
(tests/golden/e4m3_facts.json) and to torch's float8_e4m3fn casts (a library
routine); the per-row quantiser to numpy fp32 arithmetic plus those casts; the
fp8 expert to a numpy double-precision SwiGLU on the dequantised matrices; the
fp8 layer to the bf16 oracle layer when every scale is a power of two (the
dequantised weights are then exact bf16 values).
"""
import json
import os

import numpy as np
import pytest
import torch

import oracle
import synth

HERE = os.path.dirname(os.path.abspath(__file__))
FACTS = json.load(open(os.path.join(HERE, "golden", "e4m3_facts.json")))


def torch_decode(codes):
    t = torch.tensor(np.asarray(codes, np.uint8)).view(torch.float8_e4m3fn)
    return t.to(torch.float64).numpy()


def torch_encode(v):
    return torch.tensor(np.asarray(v, np.float32)).to(torch.float8_e4m3fn).view(torch.uint8).numpy()


def test_e4m3_published_constants():
    v = oracle.e4m3_values()
    assert v[FACTS["one_code"]] == 1.0
    assert v[FACTS["max_finite_code"]] == FACTS["max_finite"]
    assert np.nanmax(v) == FACTS["max_finite"] and np.nanmin(v) == -FACTS["max_finite"]
    assert v[FACTS["min_normal_code"]] == FACTS["min_normal"]
    assert v[FACTS["min_subnormal_code"]] == FACTS["min_subnormal"]
    assert sorted(np.flatnonzero(np.isnan(v)).tolist()) == FACTS["nan_codes"]
    assert int(np.isfinite(v).sum()) == FACTS["finite_codes"]
    pos = v[:128][np.isfinite(v[:128])]
    assert np.all(np.diff(pos) > 0)                       # codes 0..126 increase
    assert np.array_equal(v[128:][np.isfinite(v[128:])], -pos)   # sign bit mirrors


def test_e4m3_decode_matches_torch():
    v, t = oracle.e4m3_values(), torch_decode(np.arange(256))
    fin = np.isfinite(t)
    assert np.array_equal(np.isnan(v), np.isnan(t))
    assert np.array_equal(v[fin], t[fin])


def test_e4m3_encode_round_trip_and_saturation():
    v = oracle.e4m3_values()
    for c in range(256):
        if np.isfinite(v[c]):
            want = c
            assert oracle.e4m3_encode(v[c]) == want, c
    assert oracle.e4m3_encode(1e6) == 0x7E and oracle.e4m3_encode(-1e6) == 0xFE
    assert oracle.e4m3_encode(449.0) == 0x7E
    assert oracle.e4m3_encode(463.9) == 0x7E


def test_e4m3_ties_go_to_even():
    v = oracle.e4m3_values()
    pos = [(c, v[c]) for c in range(127)]
    for (c0, a), (c1, b) in zip(pos[:-1], pos[1:]):
        mid = np.float32((a + b) / 2)
        assert float(mid) == (a + b) / 2                   # midpoints are exact in fp32
        even = c0 if c0 % 2 == 0 else c1                   # the even mantissa (code parity)
        assert oracle.e4m3_encode(mid) == even, (c0, c1)
        assert oracle.e4m3_encode(-mid) == 0x80 | even


def test_e4m3_encode_matches_torch_in_range():
    rng = np.random.default_rng(7)
    x = np.concatenate([rng.normal(0, 1, 20000), rng.normal(0, 100, 20000),
                        rng.uniform(-448, 448, 20000), rng.normal(0, 0.003, 20000)]).astype(np.float32)
    x = x[np.abs(x) <= 448]
    mine = np.array([oracle.e4m3_encode(float(a)) for a in x], np.uint8)
    assert np.array_equal(mine, torch_encode(x))


def test_quantize_rows_matches_fp32_arithmetic():
    rng = np.random.default_rng(3)
    w = rng.normal(0, 0.02, (37, 200)).astype(np.float32)
    w[5] = 0.0                                             # all-zero row: scale 1, codes 0
    w[9, :] *= 1e-6                                        # tiny row: subnormal codes
    w[11, 17] = 3.0                                        # one outlier
    bits = synth.round_bf16(w)
    q, sc = oracle.quantize_rows_fp8(bits)
    wf = oracle.to_double(bits, "bf16").astype(np.float32)
    amax = np.abs(wf).max(axis=1)
    want_sc = np.where(amax > 0, amax / np.float32(448.0), np.float32(1.0)).astype(np.float32)
    assert np.array_equal(sc, want_sc)
    assert sc[5] == 1.0 and not q[5].any()
    want_q = torch_encode((wf / want_sc[:, None]).astype(np.float32))
    assert np.array_equal(q, want_q)
    # error bound of the dequantised weights: half a step of the code grid
    deq = oracle.dequantize_fp8(q, sc)
    step = np.maximum(np.abs(wf) * 2.0 ** -3, sc[:, None] * 2.0 ** -9)
    assert np.all(np.abs(deq - wf) <= step / 2 * (1 + 1e-6))
    # the row maximum lands on 448 * scale up to the fp32 rounding of the scale
    r = np.arange(37) != 5
    assert np.allclose(np.abs(deq[r]).max(axis=1), amax[r], rtol=2.0 ** -20)


def test_expert_ffn_fp8_matches_numpy():
    rng = np.random.default_rng(11)
    d, I = 48, 40
    def bf(a):
        return torch.tensor(a.astype(np.float32)).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    qg, sg = oracle.quantize_rows_fp8(bf(rng.normal(0, 0.2, (I, d))))
    qu, su = oracle.quantize_rows_fp8(bf(rng.normal(0, 0.2, (I, d))))
    qd, sd = oracle.quantize_rows_fp8(bf(rng.normal(0, 0.2, (d, I))))
    x = rng.normal(0, 1, d)
    dq = lambda q, s: torch_decode(q.reshape(-1)).reshape(q.shape) * s.astype(np.float64)[:, None]
    g, u = dq(qg, sg) @ x, dq(qu, su) @ x
    want = dq(qd, sd) @ (g / (1 + np.exp(-g)) * u)
    got = oracle.expert_ffn_fp8(x, qg, sg, qu, su, qd, sd)
    assert np.allclose(got, want, rtol=1e-12, atol=1e-12 * np.abs(want).max())


def test_layer_fp8_equals_bf16_layer_for_power_of_two_scales():
    cfg = synth.Config("p2", T=12, d=32, N=8, M=4, Kp=1, S=2, I=24, dtype="bf16", seed=5)
    inp = synth.layer_inputs(cfg)
    rng = np.random.default_rng(2)
    q, bf = {}, dict(inp)
    for k in ("w_gate", "w_up", "w_down", "s_gate", "s_up", "s_down"):
        shape = inp[k].shape
        codes = rng.integers(0, 256, shape).astype(np.uint8)
        codes[(codes & 0x7F) == 0x7F] = 0x3A               # no NaN codes
        scale = np.ldexp(1.0, rng.integers(-9, -4, shape[:-1])).astype(np.float32)
        q[k], q[k + "_scale"] = codes, scale
        deq = oracle.dequantize_fp8(codes, scale).astype(np.float32)
        bits = torch.tensor(deq).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
        assert np.array_equal(oracle.to_double(bits, "bf16"), oracle.dequantize_fp8(codes, scale))
        bf[k] = bits
    x = oracle.to_double(inp["x"], "bf16")
    y8, i8, w8, m8 = oracle.layer_fp8(x, inp, q, cfg.M, cfg.Kp, "bf16")
    yb, ib, wb, mb = oracle.layer(x, bf, cfg.M, cfg.Kp, "bf16")
    assert np.array_equal(i8, ib) and np.array_equal(w8, wb) and np.array_equal(m8, mb)
    assert np.array_equal(y8, yb)
