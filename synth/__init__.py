"""Seeded synthetic inputs for the MoGE layer, shared by the oracle and the CUDA path.

This module only draws numbers: it holds none of the layer's arithmetic. Both
sides of every parity check receive the very same bytes from here, generated
once on the host. The generator is counter-based (SplitMix64 + Box-Muller, see
``synth.c``), so any slice of any tensor can be produced on its own.

Workloads follow the shapes the pages give for Pangu Pro MoE (hidden size 5120,
64 routed experts in 8 groups with one expert picked per group, 4 shared
experts; "Pangu Pro MoE" summary page, section 2 and the page-4 list of the
three MoGE breakthroughs), a decode batch of 456 tokens (page 5, the official
inference report digest) and a 2 x 2048-token prefill (page 1, section 5). The
SwiGLU intermediate size 1344 and the value distributions are spec choices.
"""
from __future__ import annotations

import ctypes
import dataclasses
import os
import subprocess
from typing import Optional

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "synth.c")
_LIB = os.path.join(_HERE, "libsynth.so")

# tensor stream ids; a layer l of a stack adds 16 * l
STREAM_X, STREAM_WR, STREAM_WG, STREAM_WU, STREAM_WD = 1, 2, 3, 4, 5
STREAM_SG, STREAM_SU, STREAM_SD = 6, 7, 8
STREAM_DY = 9  # upstream gradient of the backward pass


def build(force: bool = False) -> str:
    """Compile libsynth.so next to its source (gcc, OpenMP, IEEE arithmetic)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + ".tmp%d" % os.getpid()
        subprocess.check_call(["gcc", "-O2", "-fopenmp", "-ffp-contract=off", "-fno-fast-math",
                               "-shared", "-fPIC", _SRC, "-o", tmp, "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


_lib = None


def _l():
    global _lib
    if _lib is None:
        _lib = ctypes.CDLL(build())
        u64, dbl, vp = ctypes.c_uint64, ctypes.c_double, ctypes.c_void_p
        for name in ("synth_normal_f32", "synth_normal_bf16"):
            getattr(_lib, name).argtypes = [u64, u64, u64, u64, dbl, vp]
            getattr(_lib, name).restype = None
        _lib.synth_round_bf16.argtypes = [vp, u64, vp]
        _lib.synth_round_bf16.restype = None
    return _lib


def normal(seed: int, stream: int, n: int, std: float, dtype: str, first: int = 0,
           out: Optional[np.ndarray] = None) -> np.ndarray:
    """Elements [first, first+n) of normal stream (seed, stream) scaled by std.

    dtype 'bf16' returns the raw bf16 bit patterns as uint16; 'f32' returns float32.
    """
    if dtype == "bf16":
        a = np.empty(n, np.uint16) if out is None else out
        _l().synth_normal_bf16(seed, stream, first, n, std, a.ctypes.data)
    elif dtype == "f32":
        a = np.empty(n, np.float32) if out is None else out
        _l().synth_normal_f32(seed, stream, first, n, std, a.ctypes.data)
    else:
        raise ValueError(dtype)
    return a


def round_bf16(a: np.ndarray) -> np.ndarray:
    """fp32 -> bf16 bit patterns, round to nearest even."""
    a = np.ascontiguousarray(a, dtype=np.float32)
    out = np.empty(a.shape, np.uint16)
    _l().synth_round_bf16(a.ctypes.data, a.size, out.ctypes.data)
    return out


def bf16_to_f32(a: np.ndarray) -> np.ndarray:
    """bf16 bit patterns (uint16) -> float32, exact."""
    return (a.astype(np.uint32) << 16).view(np.float32)


@dataclasses.dataclass(frozen=True)
class Config:
    """One workload: T tokens, hidden d, N routed experts in M groups, Kp picked
    per group (K = M*Kp per token), S shared experts, SwiGLU intermediate I."""
    name: str
    T: int
    d: int
    N: int
    M: int
    Kp: int
    S: int
    I: int
    dtype: str          # 'f32' or 'bf16' storage/compute type of x and weights
    seed: int
    x_std: float = 1.0
    w_std: float = 0.02
    zipf_s: float = 0.0  # > 0: per-expert router bias log(Zipf share) inside each group
    layers: int = 1

    @property
    def K(self) -> int:
        return self.M * self.Kp

    def replace(self, **kw) -> "Config":
        return dataclasses.replace(self, **kw)


CONFIGS = {
    "tiny": Config("tiny", T=64, d=256, N=16, M=4, Kp=1, S=1, I=128, dtype="f32", seed=0),
    "decode": Config("decode", T=456, d=5120, N=64, M=8, Kp=1, S=4, I=1344, dtype="bf16", seed=1),
    "prefill": Config("prefill", T=4096, d=5120, N=64, M=8, Kp=1, S=4, I=1344, dtype="bf16", seed=2),
    "skew": Config("skew", T=16384, d=5120, N=64, M=8, Kp=1, S=4, I=1344, dtype="bf16", seed=3,
                   zipf_s=1.2),
    "stack12": Config("stack12", T=456, d=5120, N=64, M=8, Kp=1, S=4, I=1344, dtype="bf16", seed=4,
                      layers=12),
}


def zipf_bias(cfg: Config) -> Optional[np.ndarray]:
    """Per-expert additive router bias for the skewed workload: inside every
    group, the expert at position j (0-based) gets log(q_{j+1}) with
    q_r proportional to r^-s, normalised over the group. None when unskewed."""
    if cfg.zipf_s <= 0:
        return None
    G = cfg.N // cfg.M
    r = np.arange(1, G + 1, dtype=np.float64)
    q = r ** (-cfg.zipf_s)
    q /= q.sum()
    return np.tile(np.log(q), cfg.M).astype(np.float32)


def layer_inputs(cfg: Config, layer: int = 0, x_stream_offset: int = 0,
                 with_x: bool = True) -> dict:
    """All inputs of one MoGE layer of ``cfg`` as host arrays.

    Layouts (row-major, nn.Linear convention [out][in]):
      x        [T][d]          w_router [N][d]        logit_bias [N] fp32 or None
      w_gate   [N][I][d]       w_up     [N][I][d]     w_down     [N][d][I]
      s_gate   [S][I][d]       s_up     [S][I][d]     s_down     [S][d][I]
    bf16 tensors are uint16 bit patterns; f32 tensors are float32.
    """
    T, d, N, S, I, dt = cfg.T, cfg.d, cfg.N, cfg.S, cfg.I, cfg.dtype
    base = 16 * layer
    out = {}
    if with_x:
        out["x"] = normal(cfg.seed, STREAM_X + base + 1000 * x_stream_offset, T * d,
                          cfg.x_std, dt).reshape(T, d)
    out["w_router"] = normal(cfg.seed, STREAM_WR + base, N * d, cfg.w_std, dt).reshape(N, d)
    out["w_gate"] = normal(cfg.seed, STREAM_WG + base, N * I * d, cfg.w_std, dt).reshape(N, I, d)
    out["w_up"] = normal(cfg.seed, STREAM_WU + base, N * I * d, cfg.w_std, dt).reshape(N, I, d)
    out["w_down"] = normal(cfg.seed, STREAM_WD + base, N * d * I, cfg.w_std, dt).reshape(N, d, I)
    out["s_gate"] = normal(cfg.seed, STREAM_SG + base, S * I * d, cfg.w_std, dt).reshape(S, I, d)
    out["s_up"] = normal(cfg.seed, STREAM_SU + base, S * I * d, cfg.w_std, dt).reshape(S, I, d)
    out["s_down"] = normal(cfg.seed, STREAM_SD + base, S * d * I, cfg.w_std, dt).reshape(S, d, I)
    out["logit_bias"] = zipf_bias(cfg)
    return out


def upstream_grad(cfg: Config, std: float = 1.0) -> np.ndarray:
    """Seeded upstream gradient dy [T][d] for the backward pass (bf16 bit
    patterns for bf16 configs, float32 otherwise)."""
    return normal(cfg.seed, STREAM_DY, cfg.T * cfg.d, std, cfg.dtype).reshape(cfg.T, cfg.d)
