"""Failure detection on the GPU without a fault: bounded device waits that can
never be satisfied (an mbarrier phase nobody completes, a completion counter
nobody increments -- the helpers every pipeline of the library waits with)
give up after their limit, the host reads MOGE_ERR_TIMEOUT through
moge_check_device_errors, the word is cleared by reading it, and the same
context then runs a layer that matches the oracle."""
import time

import numpy as np
import pytest
import torch

import mixture_grouped_experts_b200 as mg
import synth
from gpu_helpers import layer_parity

pytestmark = pytest.mark.gpu


def _clear():
    mg.lib().moge_check_device_errors(None)


def test_bounded_waits_report_timeout_and_context_survives():
    _clear()
    try:
        out = torch.full((3,), 7, dtype=torch.int32, device="cuda")
        t0 = time.perf_counter()
        mg.moge_selftest_waits(50_000, out)          # two waits of 50 ms each
        with pytest.raises(mg.MogeError) as err:
            mg.check_device_errors()
        elapsed = time.perf_counter() - t0
        assert err.value.code == mg.ERR_TIMEOUT
        assert out.cpu().tolist() == [1, 1, 0]
        assert 0.09 < elapsed < 5.0                  # both waits ran to their limit, no longer
        mg.check_device_errors()                     # reading cleared the word
    finally:
        _clear()
    cfg = synth.Config("after", T=40, d=256, N=16, M=4, Kp=1, S=1, I=192, dtype="bf16", seed=51,
                       w_std=0.05)
    layer_parity(cfg, synth.layer_inputs(cfg))
    mg.check_device_errors()
