"""Pins of the CPU oracle to things other than itself.

Each test checks the oracle against a closed form, brute force, a library
routine (numpy), or a fact the pages state (tests/golden/pages_facts.json),
chosen so that a plausible slip (softmax per group instead of global, a
transposed operand, gate and up swapped, a dropped shared expert, renormalised
weights, a wrong tie rule, an unstable dispatch order) fails at least one.
"""
import itertools
import json
import math
import os

import numpy as np
import pytest

import oracle
import synth

GOLD = json.load(open(os.path.join(os.path.dirname(__file__), "golden", "pages_facts.json")))
LN3 = math.log(3.0)
LN7 = math.log(7.0)


# --------------------------------------------------------------------------- scores
def test_softmax_is_global_closed_form():
    """Router weights zero, bias = log q: the scores are q itself, over ALL
    experts (a per-group softmax would return q renormalised per group)."""
    rng = np.random.default_rng(5)
    N, M, d = 16, 4, 8
    q = rng.dirichlet(np.ones(N))
    bias = np.log(q).astype(np.float32)
    x = rng.standard_normal((3, d))
    wr = np.zeros((N, d), np.float32)
    p = oracle.router_probs(x, wr, bias, "f32")
    assert np.allclose(p, q[None, :], rtol=2e-6, atol=0)
    assert np.allclose(p.sum(1), 1.0, atol=1e-12)


def test_equal_logits_give_uniform_scores():
    N, d = 64, 32
    x = np.random.default_rng(1).standard_normal((4, d))
    p = oracle.router_probs(x, np.zeros((N, d), np.uint16), None, "bf16")
    assert np.array_equal(p, np.full((4, N), 1.0 / N))


def test_router_dot_product_against_integer_matmul():
    """Small-integer x and router weights: the logits are exact integers that
    numpy's integer matmul gives; the oracle with (x, Wr) must equal the
    oracle with x = 0 and those logits as bias (pinned by the closed form
    above). A transposed router matrix or a wrong row stride fails."""
    rng = np.random.default_rng(7)
    T, d, N = 5, 12, 6
    xi = rng.integers(-3, 4, (T, d))
    wi = rng.integers(-3, 4, (N, d))
    logits = xi @ wi.T                       # library routine, exact
    p1 = oracle.router_probs(xi.astype(np.float64), wi.astype(np.float32), None, "f32")
    for t in range(T):
        p2 = oracle.router_probs(np.zeros((1, d)), np.zeros((N, d), np.float32),
                                 logits[t].astype(np.float32), "f32")
        assert np.allclose(p1[t], p2[0], rtol=1e-13, atol=0)


def test_bf16_weights_widen_exactly():
    vals = np.array([1.0, -2.5, 0.0078125, 3.0e-3, -7.0e5], np.float32)
    bits = synth.round_bf16(vals)
    back = synth.bf16_to_f32(bits).astype(np.float64)
    assert np.array_equal(oracle.to_double(bits, "bf16"), back)
    # bf16 is the top half of fp32: exactly representable values survive
    assert back[0] == 1.0 and back[1] == -2.5 and back[2] == 0.0078125


# --------------------------------------------------------------------------- selection
@pytest.mark.parametrize("N,M,Kp", [(16, 4, 1), (16, 4, 2), (12, 3, 2), (8, 2, 3), (6, 1, 2)])
def test_grouped_selection_brute_force(N, M, Kp):
    """Every Kp-subset of every group enumerated: the chosen subset is the one
    with the largest score sum, i.e. the in-group top-Kp."""
    rng = np.random.default_rng(N * 100 + M * 10 + Kp)
    T = 40
    p = rng.dirichlet(np.ones(N), size=T)
    idx, w, mg = oracle.select_grouped(p, M, Kp)
    G = N // M
    for t in range(T):
        for g in range(M):
            best = max(itertools.combinations(range(g * G, (g + 1) * G), Kp),
                       key=lambda s: sum(p[t, e] for e in s))
            got = idx[t, g * Kp:(g + 1) * Kp]
            assert set(got.tolist()) == set(best)
            # descending order inside the group
            assert all(p[t, got[j]] >= p[t, got[j + 1]] for j in range(Kp - 1))
        assert np.array_equal(w[t], p[t, idx[t]])          # weights = global scores, no renorm


def test_grouped_invariants_and_zero_imbalance():
    rng = np.random.default_rng(11)
    N, M, Kp, T = 64, 8, 1, 1000
    p = rng.dirichlet(np.ones(N) * 0.3, size=T)
    idx, w, mg = oracle.select_grouped(p, M, Kp)
    G = N // M
    assert np.array_equal(idx // G, np.tile(np.arange(M), (T, 1)))   # one per group, group order
    assert (w.sum(1) < 1.0).all()                                      # not renormalised
    s, loads = oracle.imbalance(idx, N, M)
    assert s == GOLD["moge_imbalance_score"]["value"] and (loads == T * Kp).all()


def test_margin_definition():
    p = np.array([[0.05, 0.30, 0.25, 0.10, 0.1, 0.2, 0.2 - 1e-9, 0.0]])
    idx, w, mg = oracle.select_grouped(p, 2, 1)
    assert idx.tolist() == [[1, 5]]
    assert mg[0] == pytest.approx(1e-9, rel=1e-6)
    # a group with every expert picked has no next candidate
    idx, w, mg = oracle.select_grouped(p, 4, 2)
    assert mg[0] == np.inf


def test_tie_goes_to_lower_index():
    p = np.array([[0.25, 0.25, 0.25, 0.25]])
    idx, _, _ = oracle.select_grouped(p, 2, 1)
    assert idx.tolist() == [[0, 2]]
    assert oracle.select_global(p, 3).tolist() == [[0, 1, 2]]


def test_one_group_is_global_topk():
    rng = np.random.default_rng(3)
    p = rng.dirichlet(np.ones(20), size=50)
    a, _, _ = oracle.select_grouped(p, 1, 5)
    b = oracle.select_global(p, 5)
    assert np.array_equal(a, b)
    ref = np.argsort(-p, axis=1, kind="stable")[:, :5]                 # library routine
    assert np.array_equal(b, ref)


def test_selection_on_logits_equals_selection_on_scores():
    rng = np.random.default_rng(9)
    x = rng.standard_normal((30, 16))
    wr = (0.3 * rng.standard_normal((16, 16))).astype(np.float32)
    p = oracle.router_probs(x, wr, None, "f32")
    logits = x @ wr.astype(np.float64).T
    a, _, _ = oracle.select_grouped(p, 4, 2)
    b, _, _ = oracle.select_grouped(logits - logits.max(1, keepdims=True) - 1.0, 4, 2)
    assert np.array_equal(a, b)


# --------------------------------------------------------------------------- imbalance
def test_imbalance_hand_cases():
    # N=4, M=2 (groups {0,1},{2,3}); T=2, K=2
    s, L = oracle.imbalance(np.array([[0, 1], [0, 2]]), 4, 2)
    assert L.tolist() == [3, 1] and s == pytest.approx(2 / 4)
    s, L = oracle.imbalance(np.array([[0, 2], [1, 3]]), 4, 2)
    assert L.tolist() == [2, 2] and s == 0.0


def test_monte_carlo_global_topk_closed_form():
    """T=1, iid scores, global top-8 of 64: P(IS = 0) = 8^8 / C(64, 8)."""
    fact = GOLD["global_top8_of_64_T1_prob_zero_imbalance"]
    assert fact["numerator"] == 8 ** 8 and fact["denominator"] == math.comb(64, 8)
    rng = np.random.default_rng(2024)
    trials = 200_000
    p = rng.random((trials, 64))
    idx = oracle.select_global(p, 8)
    zero = 0
    for chunk in np.array_split(np.arange(trials), 20):
        groups = np.sort(idx[chunk] // 8, axis=1)
        zero += int((groups == np.arange(8)).all(1).sum())
    # the oracle's score on one trial agrees with the group test
    s0, _ = oracle.imbalance(idx[:1], 64, 8)
    assert (s0 == 0.0) == bool((np.sort(idx[0] // 8) == np.arange(8)).all())
    mean = trials * fact["value"]
    sd = math.sqrt(trials * fact["value"] * (1 - fact["value"]))
    assert abs(zero - mean) < 5 * sd, (zero, mean, sd)


def test_monte_carlo_batches_imbalance():
    """Batches of 16 tokens: global top-8 is imbalanced in every trial, MoGE
    never (the pages' Monte Carlo statement)."""
    rng = np.random.default_rng(77)
    pos = 0
    for _ in range(300):
        p = rng.random((16, 64))
        sg, _ = oracle.imbalance(oracle.select_global(p, 8), 64, 8)
        sm, _ = oracle.imbalance(oracle.select_grouped(p, 8, 1)[0], 64, 8)
        pos += sg > 0
        assert sm == 0.0
    assert pos == 300


def test_within_group_share_is_one_eighth():
    rng = np.random.default_rng(8)
    T = 40_000
    p = rng.random((T, 64))
    idx, _, _ = oracle.select_grouped(p, 8, 1)
    share = np.bincount(idx.ravel(), minlength=64) / T
    target = GOLD["within_group_share_top1_of_8"]["value"]
    sd = math.sqrt(target * (1 - target) / T)
    assert np.all(np.abs(share - target) < 5 * sd)


# --------------------------------------------------------------------------- dispatch
def test_dispatch_matches_stable_sort():
    rng = np.random.default_rng(4)
    T, N, M, Kp = 97, 16, 4, 2
    p = rng.random((T, N))
    idx, _, _ = oracle.select_grouped(p, M, Kp)
    counts, offsets, ps, pd = oracle.dispatch(idx, N)
    order = np.argsort(idx.ravel(), kind="stable")                   # library routine
    assert np.array_equal(ps, order // idx.shape[1])
    assert np.array_equal(counts, np.bincount(idx.ravel(), minlength=N))
    assert np.array_equal(offsets, np.concatenate([[0], np.cumsum(counts)]))
    assert np.array_equal(pd.ravel()[order], np.arange(T * idx.shape[1]))
    G = N // M
    assert np.all(counts.reshape(M, G).sum(1) == T * Kp)             # equal group load
    for e in range(N):
        seg = ps[offsets[e]:offsets[e + 1]]
        assert np.all(np.diff(seg) > 0)                               # ascending tokens


def test_dispatch_empty_and_single_expert():
    idx = np.zeros((5, 1), np.int32) + 2
    counts, offsets, ps, pd = oracle.dispatch(idx, 4)
    assert counts.tolist() == [0, 0, 5, 0] and offsets.tolist() == [0, 0, 0, 5, 5]
    assert ps.tolist() == [0, 1, 2, 3, 4] and pd.ravel().tolist() == [0, 1, 2, 3, 4]


# --------------------------------------------------------------------------- expert FFN
def _sel(rows, cols, m, scale):
    a = np.zeros((rows, cols), np.float32)
    for r, c in enumerate(m):
        a[r, c] = scale
    return a


def test_expert_ffn_closed_form_rectangular():
    """Selection-matrix weights: gate_i = a x_{s(i)}, up_i = b x_{u(i)},
    y_o = c h_{r(o)}; silu at 0, +-ln 3 and ln 7 has the closed values
    0, 3/4 ln 3, -1/4 ln 3, 7/8 ln 7. Catches swapped gate/up (a != b), a
    transposed W_down (r not invertible), a missing silu or a sign slip."""
    d, I = 6, 4
    x = np.array([LN3, -LN3, 0.0, LN7, 2.0, -1.0])
    s_map, u_map, r_map = [0, 1, 2, 3], [4, 5, 4, 5], [3, 1, 0, 2, 2, 0]
    a, b, c = 1.0, 2.0, 0.5
    wg, wu, wd = _sel(I, d, s_map, a), _sel(I, d, u_map, b), _sel(d, I, r_map, c)
    y = oracle.expert_ffn(x, wg, wu, wd, "f32")
    silu = {0: 0.75 * LN3, 1: -0.25 * LN3, 2: 0.0, 3: 0.875 * LN7}     # silu(a x_{s(i)})
    h = [silu[i] * b * x[u_map[i]] for i in range(I)]
    ref = np.array([c * h[r_map[o]] for o in range(d)])
    assert np.allclose(y, ref, rtol=1e-14, atol=1e-15)


def test_expert_ffn_bf16_matches_f32_on_same_values():
    rng = np.random.default_rng(12)
    d, I = 16, 8
    wf = [(0.1 * rng.standard_normal(s)).astype(np.float32) for s in ((I, d), (I, d), (d, I))]
    wb = [synth.round_bf16(w) for w in wf]
    wf2 = [synth.bf16_to_f32(w) for w in wb]
    x = rng.standard_normal(d)
    assert np.array_equal(oracle.expert_ffn(x, *wb, "bf16"), oracle.expert_ffn(x, *wf2, "f32"))


def test_expert_ffn_scaling_laws():
    rng = np.random.default_rng(13)
    d, I = 24, 10
    wg, wu, wd = ((0.2 * rng.standard_normal(s)).astype(np.float32) for s in ((I, d), (I, d), (d, I)))
    x = rng.standard_normal(d)
    y = oracle.expert_ffn(x, wg, wu, wd, "f32")
    assert np.allclose(oracle.expert_ffn(x, wg, wu, 2 * wd, "f32"), 2 * y, rtol=1e-14)
    assert np.allclose(oracle.expert_ffn(x, wg, 4 * wu, wd, "f32"), 4 * y, rtol=1e-14)
    assert np.array_equal(oracle.expert_ffn(x, wg, wu, 0 * wd, "f32"), np.zeros(d))


# --------------------------------------------------------------------------- layer
def _tiny_inputs(N=8, M=2, S=1, d=12, I=6, seed=21, dtype="f32", T=10):
    cfg = synth.Config("t", T=T, d=d, N=N, M=M, Kp=1, S=S, I=I, dtype=dtype, seed=seed, w_std=0.3)
    return cfg, synth.layer_inputs(cfg)


def test_layer_all_experts_uniform_weights():
    """Kp = N/M (every expert), router weights zero: every p_e = 1/N, so
    y = (1/N) sum_e FFN_e(x) + sum_s FFN_s(x)."""
    cfg, inp = _tiny_inputs(N=8, M=2, S=2)
    inp["w_router"] = np.zeros_like(inp["w_router"])
    x = oracle.to_double(inp["x"], "f32")
    y, idx, w, _ = oracle.layer(x, inp, M=2, Kp=4, dtype="f32")
    for t in range(cfg.T):
        ref = sum(oracle.expert_ffn(x[t], inp["w_gate"][e], inp["w_up"][e], inp["w_down"][e], "f32")
                  for e in range(8)) / 8.0
        ref += sum(oracle.expert_ffn(x[t], inp["s_gate"][s], inp["s_up"][s], inp["s_down"][s], "f32")
                   for s in range(2))
        assert np.allclose(y[t], ref, rtol=1e-12, atol=1e-14)
        assert np.all(w[t] == 1.0 / 8)


def test_layer_known_scores_pick_and_weight():
    """Router zero, bias = log q: the picks are the in-group argmax of q and
    the combine weights are q at the picks (global scores, not renormalised)."""
    cfg, inp = _tiny_inputs(N=8, M=2, S=1)
    q = np.array([0.02, 0.2, 0.05, 0.03, 0.3, 0.1, 0.25, 0.05])
    inp["w_router"] = np.zeros_like(inp["w_router"])
    inp["logit_bias"] = np.log(q).astype(np.float32)
    x = oracle.to_double(inp["x"], "f32")
    y, idx, w, _ = oracle.layer(x, inp, M=2, Kp=1, dtype="f32", tokens=[3, 7])
    assert idx.tolist() == [[1, 4], [1, 4]]
    for j, t in enumerate([3, 7]):
        f = [oracle.expert_ffn(x[t], inp["w_gate"][e], inp["w_up"][e], inp["w_down"][e], "f32")
             for e in (1, 4)]
        s = oracle.expert_ffn(x[t], inp["s_gate"][0], inp["s_up"][0], inp["s_down"][0], "f32")
        assert np.allclose(w[j], q[[1, 4]], rtol=2e-6, atol=0)
        ref = w[j, 0] * f[0] + w[j, 1] * f[1] + s
        assert np.allclose(y[j], ref, rtol=1e-13, atol=1e-15)


def test_layer_shared_only_when_routed_down_is_zero():
    cfg, inp = _tiny_inputs(S=2)
    inp["w_down"] = np.zeros_like(inp["w_down"])
    x = oracle.to_double(inp["x"], "f32")
    y, _, _, _ = oracle.layer(x, inp, M=2, Kp=1, dtype="f32")
    for t in range(cfg.T):
        ref = sum(oracle.expert_ffn(x[t], inp["s_gate"][s], inp["s_up"][s], inp["s_down"][s], "f32")
                  for s in range(2))
        assert np.allclose(y[t], ref, rtol=1e-13, atol=1e-15)


def test_layer_token_permutation_equivariance():
    cfg, inp = _tiny_inputs(T=12)
    x = oracle.to_double(inp["x"], "f32")
    y, idx, _, _ = oracle.layer(x, inp, M=2, Kp=1, dtype="f32")
    perm = np.random.default_rng(0).permutation(cfg.T)
    y2, idx2, _, _ = oracle.layer(x[perm], inp, M=2, Kp=1, dtype="f32")
    assert np.array_equal(y2, y[perm]) and np.array_equal(idx2, idx[perm])
    y3, _, _, _ = oracle.layer(x, inp, M=2, Kp=1, dtype="f32", tokens=perm[:5])
    assert np.array_equal(y3, y[perm[:5]])


# --------------------------------------------------------------------------- rmsnorm
def test_rmsnorm_closed_forms():
    eps = 1e-6
    d = 64
    c = 2.5
    u = oracle.rmsnorm(np.full((1, d), c), eps)
    assert np.allclose(u, c / math.sqrt(c * c + eps), rtol=1e-15)
    x = np.random.default_rng(2).standard_normal((5, d))
    u = oracle.rmsnorm(x, eps)
    n2 = (x * x).sum(1)
    assert np.allclose((u * u).sum(1), d * n2 / (n2 + d * eps), rtol=1e-13)
    assert np.allclose(u / x, (u / x)[:, :1], rtol=1e-13)                # per-row scale only
