"""Shared helpers of the GPU parity tests: run the CUDA path through the C ABI
and compare with the oracle on the same seeded inputs.

Comparison rules (stated once, used by every GPU test):
  * routing ids / counts / permutation: bit-exact for every token whose oracle
    in-group margin (p of the Kp-th pick minus p of the best unpicked expert)
    exceeds 1e-4 in every group; a token under the margin must still hold a
    valid pick (each GPU pick scores within 1e-4 of the oracle's pick);
  * picked weights: the oracle's global softmax score at the GPU's picks, |diff| <= 1e-5;
  * layer outputs: normwise max relative error max|y - y_ref| / max|y_ref| over
    the compared rows, <= 1e-2 for bf16 layers and <= 1e-4 for fp32 layers.
"""
from __future__ import annotations

import numpy as np
import torch

import mixture_grouped_experts_b200 as mg
import oracle
import oracle_par
import synth

MARGIN = 1e-4
TOL = {"bf16": 1e-2, "f32": 1e-4}


def x_double(inp, cfg):
    return oracle.to_double(inp["x"], cfg.dtype)


def to_host_f64(t: torch.Tensor) -> np.ndarray:
    return t.float().cpu().numpy().astype(np.float64)


def normwise_err(y, ref) -> float:
    den = np.abs(ref).max()
    return float(np.abs(y - ref).max() / (den if den > 0 else 1.0))


def device_inputs(cfg, inp):
    x = mg.to_device(inp["x"], cfg.dtype)
    w = mg.weights_to_device(inp, cfg.dtype)
    return x, w


def check_routing(cfg, p_oracle, idx_o, margin_o, idx_g, w_g):
    """Compare GPU picks/weights with the oracle under the margin rule.
    Returns the boolean mask of tokens above the margin."""
    T = cfg.T
    safe = margin_o > MARGIN
    assert np.array_equal(idx_g[safe], idx_o[safe]), "routing mismatch on tokens above the margin"
    G = cfg.N // cfg.M
    # every token: Kp distinct picks per group, in its group, group-major
    grp = idx_g // G
    assert np.array_equal(grp, np.repeat(np.arange(cfg.M), cfg.Kp)[None, :].repeat(T, 0))
    for t in np.nonzero(~safe)[0]:
        for g in range(cfg.M):
            got = idx_g[t, g * cfg.Kp:(g + 1) * cfg.Kp]
            want = idx_o[t, g * cfg.Kp:(g + 1) * cfg.Kp]
            assert len(set(got.tolist())) == cfg.Kp
            assert np.all(np.abs(np.sort(p_oracle[t, got]) - np.sort(p_oracle[t, want])) <= MARGIN)
    # weights are the global scores at the picks (not renormalised)
    ref_w = np.take_along_axis(p_oracle, idx_g.astype(np.int64), axis=1)
    assert np.all(np.abs(w_g - ref_w) <= 1e-5 + 1e-4 * ref_w), float(np.abs(w_g - ref_w).max())
    return safe


def check_counts(cfg, idx_o, idx_g, counts_g, offsets_g, safe):
    """Counts of the GPU equal the histogram of its own picks (exact), the
    group loads are equal (T*Kp each), and over the tokens above the margin the
    counts equal the oracle's."""
    N = cfg.N
    assert np.array_equal(counts_g, np.bincount(idx_g.ravel(), minlength=N))
    assert offsets_g[0] == 0 and np.array_equal(np.diff(offsets_g), counts_g)
    G = N // cfg.M
    assert np.all(counts_g.reshape(cfg.M, G).sum(1) == cfg.T * cfg.Kp)
    a = np.bincount(idx_g[safe].ravel(), minlength=N)
    b = np.bincount(idx_o[safe].ravel(), minlength=N)
    assert np.array_equal(a, b)


def sample_tokens(T, n, seed=0):
    rng = np.random.default_rng(seed)
    fixed = [0, 1, T // 3, T // 2, T - 2, T - 1]
    rest = rng.choice(T, size=min(T, max(n - len(fixed), 0)), replace=False).tolist()
    out = sorted(set(t for t in fixed + rest if 0 <= t < T))
    return np.array(out[:max(n, 1)] if len(out) > n else out, dtype=np.int64)


# ------------------------------------------------------------------ oracle pool
# The oracle is single-threaded; full-size checks spread its tokens over host
# threads (oracle_par), whose ctypes calls run at once.
def _pool_workers():
    import os
    return max(1, min(8, (os.cpu_count() or 2) // 2))


def oracle_backward_pool(cfg, alpha, idx, tokens):
    """oracle.layer_backward of the seeded config `cfg` at the picks idx,
    without the routed experts' weight gradients: the token terms are split
    over host threads and summed (every gradient is a sum over tokens; the
    balance loss's f comes from the whole batch in each part)."""
    inp = synth.layer_inputs(cfg)
    xd = oracle.to_double(inp["x"], cfg.dtype)
    dy = oracle.to_double(synth.upstream_grad(cfg), cfg.dtype)
    return oracle_par.layer_backward_sum(xd, inp, cfg.M, cfg.Kp, cfg.dtype, dy, alpha, idx,
                                         tokens, _pool_workers())


def expert_tiles(rows, max_tile=256, stream_rows=64):
    """Token tiles [start, end) of an expert with `rows` rows, by the grouped
    FFN's tiling rule (one tile up to 64 rows, else ceil(rows / 256) balanced
    tiles of a multiple-of-16 width). Used to pick tokens tile by tile."""
    if rows <= 0:
        return []
    if rows <= stream_rows:
        return [(0, rows)]
    nt = -(-rows // max_tile)
    bn = (-(-rows // nt) + 15) // 16 * 16
    return [(a, min(rows, a + bn)) for a in range(0, rows, bn)]


def tile_tokens(perm_src, offsets, e, tiles):
    """Tokens held by the listed token tiles (indices into expert_tiles) of expert e."""
    out = []
    t_all = expert_tiles(int(offsets[e + 1] - offsets[e]))
    for i in tiles:
        a, b = t_all[i]
        out += perm_src[offsets[e] + a:offsets[e] + b].tolist()
    return out


def run_layer(cfg, x_dev, w_dev, ws, residual=None):
    s = mg.shape_of(cfg)
    y = mg.moge_layer_forward(s, x_dev, w_dev, ws, residual=residual)
    torch.cuda.synchronize()
    mg.check_device_errors()
    idx, wt, counts, offsets = mg.moge_workspace_routing(s, ws)
    return (y, idx.cpu().numpy(), wt.cpu().numpy().astype(np.float64), counts.cpu().numpy(),
            offsets.cpu().numpy())


def layer_parity(cfg, inp, n_sample=None, tokens=None, by_tiles=None):
    """Full layer on the GPU vs the oracle: routing of all tokens, outputs of
    sampled tokens (all tokens when n_sample is None and tokens is None).
    by_tiles (a function of (perm_src, offsets, counts) returning tokens):
    more tokens chosen from the GPU's own dispatch, every token of whole token
    tiles, run through the oracle on host threads."""
    x, w = device_inputs(cfg, inp)
    ws = mg.alloc_workspace(mg.shape_of(cfg))
    y, idx_g, w_g, counts_g, offsets_g = run_layer(cfg, x, w, ws)
    xd = x_double(inp, cfg)
    p = oracle.router_probs(xd, inp["w_router"], inp["logit_bias"], cfg.dtype)
    idx_o, w_o, mg_o = oracle.select_grouped(p, cfg.M, cfg.Kp)
    safe = check_routing(cfg, p, idx_o, mg_o, idx_g, w_g)
    check_counts(cfg, idx_o, idx_g, counts_g, offsets_g, safe)
    if tokens is None:
        tokens = np.arange(cfg.T) if n_sample is None else sample_tokens(cfg.T, n_sample)
    tokens = np.array([t for t in tokens if safe[t]], dtype=np.int64)
    y_ref, _, _, _ = oracle_par.layer(xd, inp, cfg.M, cfg.Kp, cfg.dtype, tokens=tokens)
    if by_tiles is not None:
        ps = oracle.dispatch(idx_g, cfg.N)[2]
        extra = sorted(set(int(t) for t in by_tiles(ps, offsets_g, counts_g)
                           if safe[t]) - set(tokens.tolist()))
        if extra:
            y_ref = np.concatenate([y_ref, oracle_par.layer(xd, inp, cfg.M, cfg.Kp, cfg.dtype,
                                                            tokens=extra)[0]], axis=0)
            tokens = np.concatenate([tokens, np.array(extra, dtype=np.int64)])
    y_g = to_host_f64(y)[tokens]
    err = normwise_err(y_g, y_ref)
    assert err <= TOL[cfg.dtype], (cfg.name, err)
    return dict(err=err, y=y, idx=idx_g, counts=counts_g, safe=safe, ws=ws, x=x, w=w, p=p,
                tokens=tokens)
