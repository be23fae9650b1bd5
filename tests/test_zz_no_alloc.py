"""moge_route_noalloc: routing for callers that may not allocate device memory
(for instance a plugin whose host runtime owns all device memory through its
own pool, or a serving loop that must never hit a synchronising cudaMalloc).
It keeps its scratch in a fixed array inside the library, so it must give the
same routing as moge_route with a caller workspace.

Collected last on purpose (file name): if it fails, a run that stops at the
first failure has already run every other test. It must pass alone in a fresh
process and after the other tests."""
import ctypes

import numpy as np
import pytest
import torch

import mixture_grouped_experts_b200 as mg
import synth


def _case(T, seed, N=16, M=4):
    cfg = synth.Config("noalloc", T=T, d=512, N=N, M=M, Kp=1, S=0, I=64, dtype="bf16", seed=seed)
    inp = synth.layer_inputs(cfg)
    return cfg, mg.to_device(inp["x"], "bf16"), mg.to_device(inp["w_router"], "bf16")


def _scratch_bytes(T, N, K):
    """Scratch the call needs: per-tile histograms and row bases, per-pick ranks."""
    r256 = lambda v: (v + 255) // 256 * 256
    return 2 * r256(-(-T // 16) * N * 4) + r256(T * K * 4)


@pytest.mark.gpu
def test_noalloc_route_matches_workspace_route_twice():
    # calls in a row, each larger batch before a smaller one, so that any read of
    # the previous call's leftovers in the shared array would show: a batch that
    # fills the 1 MiB array exactly (16384 tokens, 64 experts, 8 picks), one on
    # the router's 64-token tiles (>= 1024 tokens with <= 64 experts), then two
    # on its 16-token tiles
    assert _scratch_bytes(16384, 64, 8) == 1 << 20
    for T, seed, N, M in ((16384, 33, 64, 8), (1024, 34, 64, 8), (300, 31, 16, 4),
                          (77, 32, 16, 4)):
        cfg, x, wr = _case(T, seed, N, M)
        s = mg.shape_of(cfg)
        ws = mg.alloc_workspace(s)
        ref = mg.moge_route(s, x, wr, None, ws)
        got = mg.moge_route_noalloc(s, x, wr, None)
        torch.cuda.synchronize()
        mg.check_device_errors()
        names = ("topk_idx", "topk_w", "counts", "offsets", "perm_src", "perm_dst")
        for name, a, b in zip(names, ref, got):
            a, b = a.cpu().numpy(), b.cpu().numpy()
            if name == "topk_w":
                assert np.allclose(a, b, rtol=0, atol=1e-6), name
            else:
                assert np.array_equal(a, b), name
        assert int(got[2].sum()) == T * cfg.K


def test_noalloc_route_rejects_batches_above_its_scratch():
    cfg = mg.LayerShape(T=20000, d=512, N=64, M=8, Kp=1, S=0, I=64, dtype="bf16")
    rc = mg.lib().moge_route_noalloc(ctypes.byref(mg._cfg(cfg)), *([None] * 10))
    assert rc == mg.ERR_UNSUPPORTED
    assert b"1 MiB" in mg.lib().moge_last_error()
