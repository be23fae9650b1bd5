"""The oracle's per-token and per-row functions run on several host threads,
for the tests at the workloads' full sizes.

The oracle evaluates every token of a layer on its own, and quantises every
weight row on its own. These wrappers hand disjoint token lists, or disjoint
blocks of experts, to the same oracle calls on host threads, then stack the
results in the listed order. They add no arithmetic: every row is what one
sequential oracle call returns for it (the C oracle keeps no state between
calls, and its ctypes calls release the interpreter lock, so the threads run
at once). Test infrastructure only, like the oracle itself.
"""
import os
from concurrent.futures import ThreadPoolExecutor

import numpy as np

import oracle


def threads() -> int:
    return max(1, min(16, os.cpu_count() or 1))


def _load():
    """Load the oracle's library in the calling thread before any worker
    starts (its first use may compile it, which must happen once)."""
    oracle.e4m3_decode(0)


def _tokens(x, tokens):
    n = np.asarray(x).shape[0]
    return np.arange(n, dtype=np.int64) if tokens is None else np.asarray(tokens, np.int64)


def _split_tokens(fn, x, tokens, *args, **kw):
    _load()
    toks = _tokens(x, tokens)
    nt = min(threads(), len(toks))
    if nt <= 1:
        return fn(x, *args, tokens=toks, **kw)
    parts = [p for p in np.array_split(toks, nt) if len(p)]
    with ThreadPoolExecutor(len(parts)) as ex:
        outs = list(ex.map(lambda p: fn(x, *args, tokens=p, **kw), parts))
    return tuple(np.concatenate([o[i] for o in outs]) for i in range(len(outs[0])))


def layer(x, inp, M, Kp, dtype, tokens=None):
    """oracle.layer, its tokens spread over threads; same returns."""
    return _split_tokens(oracle.layer, x, tokens, inp, M, Kp, dtype)


def layer_fp8(x, inp, q, M, Kp, dtype, tokens=None):
    """oracle.layer_fp8, its tokens spread over threads; same returns."""
    return _split_tokens(oracle.layer_fp8, x, tokens, inp, q, M, Kp, dtype)


def layer_w8a8(x, inp, q, M, Kp, dtype, tokens=None):
    """oracle.layer_w8a8, its tokens spread over threads; same returns."""
    return _split_tokens(oracle.layer_w8a8, x, tokens, inp, q, M, Kp, dtype)


def quantize_experts_fp8(inp: dict) -> dict:
    """oracle.quantize_experts_fp8, each matrix's experts spread over threads
    (rows are quantised independently); same returns."""
    _load()
    jobs = []
    for k in ("w_gate", "w_up", "w_down", "s_gate", "s_up", "s_down"):
        w = inp[k]
        for blk in np.array_split(np.arange(w.shape[0]), min(threads(), max(1, w.shape[0]))):
            if len(blk):
                jobs.append((k, blk[0], blk[-1] + 1))
    with ThreadPoolExecutor(threads()) as ex:
        res = list(ex.map(lambda j: oracle.quantize_rows_fp8(inp[j[0]][j[1]:j[2]]), jobs))
    out = {}
    for k in ("w_gate", "w_up", "w_down", "s_gate", "s_up", "s_down"):
        got = [r for j, r in zip(jobs, res) if j[0] == k]
        if got:
            out[k] = np.concatenate([g[0] for g in got])
            out[k + "_scale"] = np.concatenate([g[1] for g in got])
        else:   # no expert of this kind (S = 0)
            out[k], out[k + "_scale"] = oracle.quantize_rows_fp8(inp[k])
    return out


def layer_backward_sum(x, inp, M, Kp, dtype, dy, alpha, idx, tokens, parts):
    """oracle.layer_backward without the routed experts' weight gradients,
    its token terms split into `parts` lists on threads and summed in list
    order (every gradient is a sum over tokens; the balance loss's batch
    shares come from the whole batch in every part, so aux is part 0's)."""
    _load()
    toks = _tokens(x, tokens)
    chunks = [c for c in np.array_split(toks, max(1, min(parts, len(toks)))) if len(c)] or [toks]
    with ThreadPoolExecutor(len(chunks)) as ex:
        outs = list(ex.map(lambda c: oracle.layer_backward(x, inp, M, Kp, dtype, dy, alpha,
                                                           idx=idx, tokens=c,
                                                           routed_weights=False), chunks))
    out = {k: sum(o[k] for o in outs) for k in outs[0] if k != "aux"}
    out["aux"] = outs[0]["aux"]
    return out
