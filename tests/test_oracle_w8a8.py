"""Pins of the oracle's W8A8 functions: 8-bit weights and activations quantised
per token (CPU only).

* The activation quantiser is pinned to numpy fp32 arithmetic for the scale
  and to torch's float8_e4m3fn casts (a library routine) for the codes. On
  bf16 rows it must also agree with the weight quantiser, which is pinned in
  test_oracle_fp8.py.
* The W8A8 expert is pinned to the weights-only 8-bit expert (pinned in
  test_oracle_fp8.py) through two special cases:
  - With one intermediate feature (I = 1), quantising h loses nothing but
    fp32 rounding: the row scale maps the lone value to +-448 exactly. The two
    experts then agree on x whose quantisation is lossless.
  - With W_down a permutation matrix, the output is the quantised h, permuted.
    It must equal the activation quantiser applied to the weights-only
    expert's output, after x is replaced by its dequantised 8-bit form.
* The W8A8 layer is pinned through two checks:
  - It combines W8A8 experts with the routing and combine rule of the pinned
    layers.
  - At I = 1 with lossless x it agrees with the weights-only 8-bit layer.
"""
import numpy as np
import torch

import oracle
import synth

from test_oracle_fp8 import torch_encode


def _bf16_bits(a):
    return torch.tensor(np.asarray(a, np.float32)).to(torch.bfloat16).view(torch.int16).numpy() \
        .view(np.uint16)


def _expected_act_quant(v):
    v32 = np.asarray(v, np.float64).astype(np.float32)
    amax = np.abs(v32).max(axis=-1)
    scale = np.where(amax > 0, amax / np.float32(448.0), np.float32(1.0)).astype(np.float32)
    q = torch_encode(v32 / scale[..., None])
    return q, scale


def test_act_quantiser_matches_fp32_arithmetic_and_torch_casts():
    rng = np.random.default_rng(11)
    rows = rng.standard_normal((40, 96)) * np.exp(rng.uniform(-12, 12, (40, 1)))
    rows[3] = 0.0                                    # all-zero row: scale 1, codes 0
    rows[5, :] = rng.standard_normal(96) * 1e-30     # tiny values: scale in fp32's normal range
    rows[7, 0] = 1e4                                 # one large value: the rest E4M3-subnormal
    rows[9] = np.linspace(-3.0, 3.0, 96)             # evenly spaced values
    q, s = oracle.quantize_act_rows(rows)
    q_want, s_want = _expected_act_quant(rows)
    assert np.array_equal(s, s_want)
    assert np.array_equal(q, q_want)
    assert s[3] == 1.0 and not q[3].any()
    # every row's largest magnitude lands on +-448 (code 0x7E / 0xFE)
    nz = np.abs(rows).max(axis=1) > 0
    assert np.all((q[nz] & 0x7F).max(axis=1) == 0x7E)


def test_act_quantiser_on_bf16_rows_is_the_weight_quantiser():
    rng = np.random.default_rng(12)
    bits = _bf16_bits(rng.standard_normal((24, 80)).astype(np.float32) * 0.05)
    vals = torch.tensor(bits.view(np.int16)).view(torch.bfloat16).to(torch.float64).numpy()
    qa, sa = oracle.quantize_act_rows(vals)
    qw, sw = oracle.quantize_rows_fp8(bits)
    assert np.array_equal(qa, qw) and np.array_equal(sa, sw)


def _fp8_expert(rng, d, I, wd=None):
    def q(shape, std):
        return oracle.quantize_rows_fp8(_bf16_bits(rng.standard_normal(shape) * std))
    qg, sg = q((I, d), 0.2)
    qu, su = q((I, d), 0.2)
    if wd is None:
        qd, sd = q((d, I), 0.2)
    else:
        qd, sd = oracle.quantize_rows_fp8(_bf16_bits(wd))
    return qg, sg, qu, su, qd, sd


def _lossless_x(rng, d, shift=-5):
    """x whose 8-bit quantisation is exact: E4M3 values times 2^shift with a
    +-448 element, so the row scale is 2^shift and every code is exact."""
    finite = [c for c in range(256) if c not in (0x7F, 0xFF)]
    codes = rng.choice(finite, d).astype(np.uint8)
    codes[rng.integers(d)] = 0x7E if rng.random() < 0.5 else 0xFE
    x = oracle.e4m3_values()[codes] * 2.0 ** shift
    q, s = oracle.quantize_act_rows(x)
    assert s == np.float32(2.0 ** shift) and np.array_equal(q, codes)
    return x


def test_w8a8_expert_equals_weights_only_expert_when_quantisation_is_lossless():
    rng = np.random.default_rng(13)
    for d in (16, 48, 200):
        e = _fp8_expert(rng, d, 1)
        for _ in range(3):
            x = _lossless_x(rng, d)
            y8 = oracle.expert_ffn_w8a8(x, *e)
            y16 = oracle.expert_ffn_fp8(x, *e)
            assert np.abs(y8 - y16).max() <= 1e-6 * np.abs(y16).max(), d


def test_w8a8_expert_with_permutation_down_projection_is_the_quantised_h():
    rng = np.random.default_rng(14)
    for n in (24, 64):
        d = I = n
        perm = rng.permutation(n)
        while np.any(perm[perm] == np.arange(n)):    # no fixed points of perm o perm:
            perm = rng.permutation(n)                # a transposed W_down would differ
        wd = np.zeros((n, n), np.float32)
        wd[np.arange(n), perm] = 1.0                 # y[o] = h[perm[o]]
        e = _fp8_expert(rng, d, I, wd)
        w1 = 448.0 * float(e[5][0])                  # every dequantised 1.0: 448 * fp32(1/448)
        for x in (_lossless_x(rng, d), rng.standard_normal(d) * 0.7):
            # the weights-only expert on x's dequantised 8-bit form gives w1 * h[perm]
            qx, sx = oracle.quantize_act_rows(x)
            x_deq = oracle.e4m3_values()[qx] * float(sx)
            h_perm = oracle.expert_ffn_fp8(x_deq, *e) / w1
            qh, sh = oracle.quantize_act_rows(h_perm)
            want = oracle.e4m3_values()[qh] * float(sh) * w1
            got = oracle.expert_ffn_w8a8(x, *e)
            assert np.abs(got - want).max() <= 1e-12 * np.abs(want).max(), n
            # and the quantisation of h is visible: not the unquantised expert
            assert np.abs(got - oracle.expert_ffn_fp8(x_deq, *e)).max() > 1e-4 * np.abs(want).max()


def _quantised(inp):
    return oracle.quantize_experts_fp8(inp)


def test_w8a8_layer_combines_w8a8_experts_by_the_routing():
    cfg = synth.Config("w8a8_pin", T=6, d=32, N=8, M=2, Kp=2, S=2, I=16, dtype="bf16", seed=15,
                       w_std=0.1)
    inp = synth.layer_inputs(cfg)
    q = _quantised(inp)
    x = oracle.to_double(inp["x"], cfg.dtype)
    y, idx, w, _ = oracle.layer_w8a8(x, inp, q, cfg.M, cfg.Kp, cfg.dtype)
    _, idx_r, w_r, _ = oracle.layer(x, inp, cfg.M, cfg.Kp, cfg.dtype)
    assert np.array_equal(idx, idx_r) and np.array_equal(w, w_r)

    def ex(t, side, e):
        k = "w" if side == "w" else "s"
        return oracle.expert_ffn_w8a8(x[t], q[k + "_gate"][e], q[k + "_gate_scale"][e],
                                      q[k + "_up"][e], q[k + "_up_scale"][e],
                                      q[k + "_down"][e], q[k + "_down_scale"][e])
    for t in range(cfg.T):
        want = sum(w[t, k] * ex(t, "w", idx[t, k]) for k in range(idx.shape[1]))
        want = want + sum(ex(t, "s", s) for s in range(cfg.S))
        assert np.abs(y[t] - want).max() <= 1e-12 * np.abs(want).max()


def test_w8a8_layer_equals_weights_only_layer_when_quantisation_is_lossless():
    cfg = synth.Config("w8a8_pin1", T=8, d=48, N=8, M=4, Kp=1, S=1, I=1, dtype="bf16", seed=16,
                       w_std=0.1)
    inp = synth.layer_inputs(cfg)
    q = _quantised(inp)
    rng = np.random.default_rng(16)
    x = np.stack([_lossless_x(rng, cfg.d, shift=-8) for _ in range(cfg.T)])
    y8, idx8, _, _ = oracle.layer_w8a8(x, inp, q, cfg.M, cfg.Kp, cfg.dtype)
    y16, idx16, _, _ = oracle.layer_fp8(x, inp, q, cfg.M, cfg.Kp, cfg.dtype)
    assert np.array_equal(idx8, idx16)
    assert np.abs(y8 - y16).max() <= 1e-6 * np.abs(y16).max()
