"""CPU oracle of the MoGE layer forward and backward (fp64, single thread, plain C in oracle.c).

TEST INFRASTRUCTURE ONLY: the tests, the package smoke check and the benchmark's
CPU-baseline leg use it; the product path never imports it. It shares no code
with the CUDA library; both sides only share the seeded inputs of ``synth``.

Functions with no independent pin are listed in the header of oracle.c and in
the design notes ("parity unpinned"); every function here is pinned by
tests/test_oracle.py against closed forms, brute force or library routines.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from typing import Optional, Sequence

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")

F32, BF16 = 0, 1
_DT = {"f32": F32, "bf16": BF16}


def compile_lib(src: str, out: str) -> str:
    """gcc -O2, strict IEEE double (no contraction, no fast math), shared library."""
    tmp = out + ".tmp%d" % os.getpid()
    subprocess.check_call(["gcc", "-O2", "-std=c11", "-ffp-contract=off", "-fno-fast-math",
                           "-shared", "-fPIC", src, "-o", tmp, "-lm"])
    os.replace(tmp, out)
    return out


def build(force: bool = False) -> str:
    """Compile liboracle.so (one thread). The environment variable
    ORACLE_LIB names another build of oracle.c to load instead; only the
    planted-mistake tests set it (tests/test_oracle_plants.py)."""
    override = os.environ.get("ORACLE_LIB")
    if override:
        return override
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        compile_lib(_SRC, _LIB)
    return _LIB


_lib = None


def _l():
    global _lib
    if _lib is None:
        lib = ctypes.CDLL(build())
        vp, i32 = ctypes.c_void_p, ctypes.c_int
        lib.oracle_router_probs.argtypes = [vp, vp, vp, i32, i32, i32, i32, vp]
        lib.oracle_select_grouped.argtypes = [vp, i32, i32, i32, i32, vp, vp, vp]
        lib.oracle_select_global.argtypes = [vp, i32, i32, i32, vp]
        lib.oracle_route.argtypes = [vp, vp, vp, i32, i32, i32, i32, i32, i32, vp, vp, vp]
        lib.oracle_imbalance.argtypes = [vp, i32, i32, i32, i32, vp]
        lib.oracle_imbalance.restype = ctypes.c_double
        lib.oracle_dispatch.argtypes = [vp, i32, i32, i32, vp, vp, vp, vp]
        lib.oracle_expert_ffn.argtypes = [vp, vp, vp, vp, i32, i32, i32, vp]
        lib.oracle_layer.argtypes = [vp, i32, i32, i32, i32, i32, i32, i32, i32,
                                     vp, vp, vp, vp, vp, vp, vp, vp, vp, i32, vp, vp, vp, vp]
        lib.oracle_rmsnorm.argtypes = [vp, i32, i32, ctypes.c_double, vp]
        lib.oracle_e4m3_decode.argtypes = [ctypes.c_uint8]
        lib.oracle_e4m3_decode.restype = ctypes.c_double
        lib.oracle_e4m3_encode.argtypes = [ctypes.c_float]
        lib.oracle_e4m3_encode.restype = ctypes.c_uint8
        i64 = ctypes.c_int64
        lib.oracle_quantize_rows_fp8.argtypes = [vp, i64, i64, vp, vp]
        lib.oracle_expert_ffn_fp8.argtypes = [vp, vp, vp, vp, vp, vp, vp, i32, i32, vp]
        lib.oracle_layer_fp8.argtypes = [vp, i32, i32, i32, i32, i32, i32, i32, i32, vp, vp,
                                         vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp,
                                         vp, i32, vp, vp, vp, vp]
        lib.oracle_quantize_act_rows.argtypes = [vp, i64, i64, vp, vp]
        lib.oracle_expert_ffn_w8a8.argtypes = [vp, vp, vp, vp, vp, vp, vp, i32, i32, vp]
        lib.oracle_layer_w8a8.argtypes = lib.oracle_layer_fp8.argtypes
        lib.oracle_layer_backward.argtypes = [vp, i32, i32, i32, i32, i32, i32, i32, i32,
                                              vp, vp, vp, vp, vp, vp, vp, vp, vp,
                                              ctypes.c_double, vp, vp, i32, vp, vp, vp, vp, vp,
                                              vp, vp, vp, vp]
        lib.oracle_layer_ep_partial.argtypes = [vp, i32, i32, i32, i32, i32, i32, i32, i32, vp, vp,
                                                i32, i32, vp, vp, vp, i32, vp, vp, vp, vp, i32, vp]
        lib.oracle_expert_backward.argtypes = [vp, vp, vp, i32, vp, vp, vp, i32, i32, i32, vp, vp,
                                               vp]
        _lib = lib
    return _lib


def _p(a: Optional[np.ndarray]):
    return None if a is None else a.ctypes.data


def _chk(rc: int, what: str):
    if rc != 0:
        raise ValueError("oracle %s failed (code %d)" % (what, rc))


def to_double(a: np.ndarray, dtype: str) -> np.ndarray:
    """Widen stored values (bf16 bit patterns or float32) to float64 exactly."""
    if dtype == "bf16":
        return (a.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    return np.asarray(a, dtype=np.float32).astype(np.float64)


def _w(a: np.ndarray, dtype: str) -> np.ndarray:
    want = np.uint16 if dtype == "bf16" else np.float32
    if a.dtype != want:
        raise TypeError("weights must be %s for dtype %s" % (want, dtype))
    return np.ascontiguousarray(a)


def router_probs(x: np.ndarray, w_router: np.ndarray, bias: Optional[np.ndarray],
                 dtype: str) -> np.ndarray:
    """Global softmax scores p [T][N] (x given as float64 [T][d])."""
    x = np.ascontiguousarray(x, np.float64)
    wr = _w(w_router, dtype)
    T, d = x.shape
    N = wr.shape[0]
    b = None if bias is None else np.ascontiguousarray(bias, np.float32)
    p = np.empty((T, N), np.float64)
    _chk(_l().oracle_router_probs(_p(x), _p(wr), _p(b), _DT[dtype], T, d, N, _p(p)), "router_probs")
    return p


def select_grouped(p: np.ndarray, M: int, Kp: int):
    """Per-group top-Kp on scores p [T][N] -> (idx [T][M*Kp] int32, w float64, margin [T])."""
    p = np.ascontiguousarray(p, np.float64)
    T, N = p.shape
    idx = np.empty((T, M * Kp), np.int32)
    w = np.empty((T, M * Kp), np.float64)
    mg = np.empty(T, np.float64)
    _chk(_l().oracle_select_grouped(_p(p), T, N, M, Kp, _p(idx), _p(w), _p(mg)), "select_grouped")
    return idx, w, mg


def select_global(p: np.ndarray, K: int) -> np.ndarray:
    """Conventional global top-K on scores p [T][N] -> idx [T][K]."""
    p = np.ascontiguousarray(p, np.float64)
    T, N = p.shape
    idx = np.empty((T, K), np.int32)
    _chk(_l().oracle_select_global(_p(p), T, N, K, _p(idx)), "select_global")
    return idx


def route(x: np.ndarray, w_router: np.ndarray, bias, dtype: str, M: int, Kp: int):
    """Scores + group-balanced selection for a batch -> (idx, w, margin)."""
    x = np.ascontiguousarray(x, np.float64)
    wr = _w(w_router, dtype)
    T, d = x.shape
    N = wr.shape[0]
    b = None if bias is None else np.ascontiguousarray(bias, np.float32)
    idx = np.empty((T, M * Kp), np.int32)
    w = np.empty((T, M * Kp), np.float64)
    mg = np.empty(T, np.float64)
    _chk(_l().oracle_route(_p(x), _p(wr), _p(b), _DT[dtype], T, d, N, M, Kp,
                           _p(idx), _p(w), _p(mg)), "route")
    return idx, w, mg


def imbalance(idx: np.ndarray, N: int, M: int):
    """(imbalance score, per-group loads [M]) of an assignment matrix [T][K]."""
    idx = np.ascontiguousarray(idx, np.int32)
    T, K = idx.shape
    loads = np.empty(M, np.int64)
    s = _l().oracle_imbalance(_p(idx), T, K, N, M, _p(loads))
    return float(s), loads


def dispatch(idx: np.ndarray, N: int):
    """(counts [N], offsets [N+1], perm_src [T*K], perm_dst [T][K]) of idx [T][K]."""
    idx = np.ascontiguousarray(idx, np.int32)
    T, K = idx.shape
    counts = np.empty(N, np.int32)
    offsets = np.empty(N + 1, np.int32)
    ps = np.empty(T * K, np.int32)
    pd = np.empty((T, K), np.int32)
    _chk(_l().oracle_dispatch(_p(idx), T, K, N, _p(counts), _p(offsets), _p(ps), _p(pd)), "dispatch")
    return counts, offsets, ps, pd


def expert_ffn(x_row: np.ndarray, wg: np.ndarray, wu: np.ndarray, wd: np.ndarray,
               dtype: str) -> np.ndarray:
    """One SwiGLU expert on one token (x_row float64 [d]; wg,wu [I][d]; wd [d][I])."""
    x = np.ascontiguousarray(x_row, np.float64)
    wg, wu, wd = _w(wg, dtype), _w(wu, dtype), _w(wd, dtype)
    I, d = wg.shape
    y = np.empty(d, np.float64)
    _chk(_l().oracle_expert_ffn(_p(x), _p(wg), _p(wu), _p(wd), _DT[dtype], d, I, _p(y)), "expert_ffn")
    return y


def layer(x: np.ndarray, inp: dict, M: int, Kp: int, dtype: str,
          tokens: Optional[Sequence[int]] = None):
    """MoGE layer output for the listed tokens (all when None).

    x: float64 [T][d]; inp: the weight dict of synth.layer_inputs.
    Returns (y [n][d] float64, idx [n][K], w [n][K], margin [n]).
    """
    x = np.ascontiguousarray(x, np.float64)
    T, d = x.shape
    wr = _w(inp["w_router"], dtype)
    wg, wu, wd = _w(inp["w_gate"], dtype), _w(inp["w_up"], dtype), _w(inp["w_down"], dtype)
    N, I = wg.shape[0], wg.shape[1]
    S = inp["s_gate"].shape[0]
    sg, su, sd = (_w(inp[k], dtype) if S > 0 else None for k in ("s_gate", "s_up", "s_down"))
    b = inp.get("logit_bias")
    b = None if b is None else np.ascontiguousarray(b, np.float32)
    toks = np.arange(T, dtype=np.int32) if tokens is None else np.asarray(tokens, np.int32)
    n = len(toks)
    K = M * Kp
    y = np.empty((n, d), np.float64)
    idx = np.empty((n, K), np.int32)
    w = np.empty((n, K), np.float64)
    mg = np.empty(n, np.float64)
    _chk(_l().oracle_layer(_p(x), T, d, N, M, Kp, S, I, _DT[dtype], _p(wr), _p(b),
                           _p(wg), _p(wu), _p(wd), _p(sg), _p(su), _p(sd),
                           _p(toks), n, _p(y), _p(idx), _p(w), _p(mg)), "layer")
    return y, idx, w, mg


def layer_backward(x: np.ndarray, inp: dict, M: int, Kp: int, dtype: str, dy: np.ndarray,
                   alpha: float = 0.0, idx: Optional[np.ndarray] = None,
                   tokens: Optional[Sequence[int]] = None, weights: bool = True,
                   routed_weights: bool = True) -> dict:
    """Gradients of sum_t dy_t . y_t + L_aux (routing held fixed) -- oracle.c,
    oracle_layer_backward. x, dy: float64 [T][d]; idx: optional picks [T][M*Kp]
    to hold the routing at (default: the oracle's own); tokens: only these
    tokens' terms (their dx rows exact, weight gradients partial); weights=False:
    dx alone (no weight-gradient arrays, for full-size samples); routed_weights=False:
    the router's and the shared experts' weight gradients but not the routed
    experts' (whose arrays are the large ones). Returns float64 arrays
    dx [T][d], w_router [N][d], w_gate/w_up [N][I][d], w_down [N][d][I],
    s_gate/s_up [S][I][d], s_down [S][d][I], and the scalar aux."""
    x = np.ascontiguousarray(x, np.float64)
    dy = np.ascontiguousarray(dy, np.float64)
    T, d = x.shape
    wr = _w(inp["w_router"], dtype)
    wg, wu, wd = _w(inp["w_gate"], dtype), _w(inp["w_up"], dtype), _w(inp["w_down"], dtype)
    N, I = wg.shape[0], wg.shape[1]
    S = inp["s_gate"].shape[0]
    sg, su, sd = (_w(inp[k], dtype) if S > 0 else None for k in ("s_gate", "s_up", "s_down"))
    b = inp.get("logit_bias")
    b = None if b is None else np.ascontiguousarray(b, np.float32)
    out = {"dx": np.empty((T, d))}
    if weights:
        out.update({"w_router": np.empty((N, d)), "s_gate": np.empty((S, I, d)),
                    "s_up": np.empty((S, I, d)), "s_down": np.empty((S, d, I))})
        if routed_weights:
            out.update({"w_gate": np.empty((N, I, d)), "w_up": np.empty((N, I, d)),
                        "w_down": np.empty((N, d, I))})
    aux = np.zeros(1)
    picks = None if idx is None else np.ascontiguousarray(idx, np.int32)
    toks = None if tokens is None else np.ascontiguousarray(tokens, np.int32)
    _chk(_l().oracle_layer_backward(_p(x), T, d, N, M, Kp, S, I, _DT[dtype], _p(wr), _p(b),
                                    _p(wg), _p(wu), _p(wd), _p(sg), _p(su), _p(sd), _p(dy),
                                    float(alpha), _p(picks), _p(toks), 0 if toks is None else len(toks),
                                    _p(out["dx"]), *[_p(out.get(k)) for k in
                                                     ("w_router", "w_gate", "w_up", "w_down",
                                                      "s_gate", "s_up", "s_down")],
                                    _p(aux)), "layer_backward")
    out["aux"] = float(aux[0])
    return out


def expert_backward(x_rows: np.ndarray, dy_rows: np.ndarray, w: np.ndarray, wg: np.ndarray,
                    wu: np.ndarray, wd: np.ndarray, dtype: str):
    """One expert's weight gradients from the tokens that chose it (oracle.c,
    oracle_expert_backward): x_rows, dy_rows float64 [n][d], w [n] the tokens'
    routing weights. Returns (dw_gate [I][d], dw_up [I][d], dw_down [d][I])."""
    x_rows = np.ascontiguousarray(x_rows, np.float64)
    dy_rows = np.ascontiguousarray(dy_rows, np.float64)
    w = np.ascontiguousarray(w, np.float64)
    wg, wu, wd = _w(wg, dtype), _w(wu, dtype), _w(wd, dtype)
    I, d = wg.shape
    dwg, dwu, dwd = np.empty((I, d)), np.empty((I, d)), np.empty((d, I))
    _chk(_l().oracle_expert_backward(_p(x_rows), _p(dy_rows), _p(w), len(w), _p(wg), _p(wu),
                                     _p(wd), _DT[dtype], d, I, _p(dwg), _p(dwu), _p(dwd)),
         "expert_backward")
    return dwg, dwu, dwd


def layer_ep_partial(x: np.ndarray, w_router: np.ndarray, bias: Optional[np.ndarray], e0: int,
                     routed: Sequence[np.ndarray], shared: Sequence[np.ndarray], N: int, M: int,
                     Kp: int, dtype: str, tokens: Optional[Sequence[int]] = None) -> np.ndarray:
    """One rank's share of the layer (oracle.c, oracle_layer_ep_partial): the
    router over all N experts; routed = (w_gate, w_up, w_down) of experts
    [e0, e0 + n_loc) only; shared = (s_gate [S][I_s][d], s_up, s_down [S][d][I_s])
    slices (S may be 0). Returns y [n][d] float64 for the listed tokens."""
    x = np.ascontiguousarray(x, np.float64)
    T, d = x.shape
    wr = _w(w_router, dtype)
    wg, wu, wd = (_w(a, dtype) for a in routed)
    n_loc, I = wg.shape[0], wg.shape[1]
    sg, su, sd = (_w(a, dtype) for a in shared)
    S, I_s = sg.shape[0], sg.shape[1]
    b = None if bias is None else np.ascontiguousarray(bias, np.float32)
    toks = np.arange(T, dtype=np.int32) if tokens is None else np.asarray(tokens, np.int32)
    y = np.empty((len(toks), d))
    _chk(_l().oracle_layer_ep_partial(_p(x), T, d, N, M, Kp, S, I, _DT[dtype], _p(wr), _p(b), e0,
                                      n_loc, _p(wg), _p(wu), _p(wd), I_s, _p(sg), _p(su), _p(sd),
                                      _p(toks), len(toks), _p(y)), "layer_ep_partial")
    return y


def rmsnorm(x: np.ndarray, eps: float = 1e-6) -> np.ndarray:
    """u = x / sqrt(mean(x^2) + eps), unit gain, per row."""
    x = np.ascontiguousarray(x, np.float64)
    T, d = x.shape
    u = np.empty_like(x)
    _chk(_l().oracle_rmsnorm(_p(x), T, d, eps, _p(u)), "rmsnorm")
    return u


# ----------------------------------------------------------------------------- fp8 weights
def e4m3_decode(code: int) -> float:
    """Value of one OCP FP8 E4M3 code (NaN for S.1111.111)."""
    return float(_l().oracle_e4m3_decode(int(code) & 0xFF))


def e4m3_encode(v: float) -> int:
    """Nearest E4M3 code to the fp32 value v (ties to even, saturating at 448)."""
    return int(_l().oracle_e4m3_encode(float(np.float32(v))))


def e4m3_values() -> np.ndarray:
    """Values of all 256 codes (float64; NaN at 0x7F and 0xFF)."""
    return np.array([e4m3_decode(c) for c in range(256)], np.float64)


def quantize_rows_fp8(w: np.ndarray):
    """Per-row fp8 quantisation of bf16 rows (uint16 bit patterns, [..., cols]).

    Returns (q uint8 of the same shape, scale float32 of shape w.shape[:-1]):
    scale = amax / 448 in fp32 (1 for an all-zero row), q = E4M3(fp32(w / scale)).
    """
    w = np.ascontiguousarray(w)
    if w.dtype != np.uint16:
        raise TypeError("quantize_rows_fp8 takes bf16 bit patterns (uint16)")
    cols = w.shape[-1]
    rows = w.size // cols
    q = np.empty(w.shape, np.uint8)
    sc = np.empty(w.shape[:-1], np.float32)
    _chk(_l().oracle_quantize_rows_fp8(_p(w), rows, cols, _p(q), _p(sc)), "quantize_rows_fp8")
    return q, sc


def dequantize_fp8(q: np.ndarray, scale: np.ndarray) -> np.ndarray:
    """decode(q) * scale per row, float64 (exact)."""
    return e4m3_values()[q] * np.asarray(scale, np.float64)[..., None]


def quantize_experts_fp8(inp: dict) -> dict:
    """Quantise every expert matrix of a synth.layer_inputs weight dict (bf16)."""
    out = {}
    for k in ("w_gate", "w_up", "w_down", "s_gate", "s_up", "s_down"):
        out[k], out[k + "_scale"] = quantize_rows_fp8(inp[k])
    return out


def expert_ffn_fp8(x_row: np.ndarray, qg, sg, qu, su, qd, sd) -> np.ndarray:
    """One SwiGLU expert on one token with fp8 weights (qg, qu [I][d]; qd [d][I])."""
    x = np.ascontiguousarray(x_row, np.float64)
    qg, qu, qd = (np.ascontiguousarray(a, np.uint8) for a in (qg, qu, qd))
    sg, su, sd = (np.ascontiguousarray(a, np.float32) for a in (sg, su, sd))
    I, d = qg.shape
    y = np.empty(d, np.float64)
    _chk(_l().oracle_expert_ffn_fp8(_p(x), _p(qg), _p(sg), _p(qu), _p(su), _p(qd), _p(sd),
                                    d, I, _p(y)), "expert_ffn_fp8")
    return y


def quantize_act_rows(v: np.ndarray):
    """Per-row 8-bit activation quantisation (the W8A8 reading): each row of
    v (any float dtype, [..., cols]) is taken in fp32, then scale = amax / 448
    in fp32 (1 for an all-zero row) and q = E4M3(fp32(v / scale)).
    Returns (q uint8 of v's shape, scale float32 of shape v.shape[:-1])."""
    v = np.ascontiguousarray(v, np.float64)
    cols = v.shape[-1]
    rows = v.size // cols
    q = np.empty(v.shape, np.uint8)
    sc = np.empty(v.shape[:-1], np.float32)
    _chk(_l().oracle_quantize_act_rows(_p(v), rows, cols, _p(q), _p(sc)), "quantize_act_rows")
    return q, sc


def expert_ffn_w8a8(x_row: np.ndarray, qg, sg, qu, su, qd, sd) -> np.ndarray:
    """One SwiGLU expert on one token in W8A8: fp8 weights (qg, qu [I][d]; qd
    [d][I]) and x, h quantised per token before their products."""
    x = np.ascontiguousarray(x_row, np.float64)
    qg, qu, qd = (np.ascontiguousarray(a, np.uint8) for a in (qg, qu, qd))
    sg, su, sd = (np.ascontiguousarray(a, np.float32) for a in (sg, su, sd))
    I, d = qg.shape
    y = np.empty(d, np.float64)
    _chk(_l().oracle_expert_ffn_w8a8(_p(x), _p(qg), _p(sg), _p(qu), _p(su), _p(qd), _p(sd),
                                     d, I, _p(y)), "expert_ffn_w8a8")
    return y


def layer_w8a8(x: np.ndarray, inp: dict, q: dict, M: int, Kp: int, dtype: str,
               tokens: Optional[Sequence[int]] = None):
    """MoGE layer output in W8A8 (fp8 expert weights q in quantize_experts_fp8
    form, activations quantised per token); router from inp. Same returns as layer()."""
    return layer_fp8(x, inp, q, M, Kp, dtype, tokens, _act8=True)


def layer_fp8(x: np.ndarray, inp: dict, q: dict, M: int, Kp: int, dtype: str,
              tokens: Optional[Sequence[int]] = None, _act8: bool = False):
    """MoGE layer output with fp8 expert weights q (quantize_experts_fp8 form);
    router weights and logit bias from inp. Same returns as layer()."""
    x = np.ascontiguousarray(x, np.float64)
    T, d = x.shape
    wr = _w(inp["w_router"], dtype)
    N, I = q["w_gate"].shape[0], q["w_gate"].shape[1]
    S = q["s_gate"].shape[0]
    a = {k: np.ascontiguousarray(v) for k, v in q.items()}
    b = inp.get("logit_bias")
    b = None if b is None else np.ascontiguousarray(b, np.float32)
    toks = np.arange(T, dtype=np.int32) if tokens is None else np.asarray(tokens, np.int32)
    n = len(toks)
    K = M * Kp
    y = np.empty((n, d), np.float64)
    idx = np.empty((n, K), np.int32)
    w = np.empty((n, K), np.float64)
    mg = np.empty(n, np.float64)
    fn = _l().oracle_layer_w8a8 if _act8 else _l().oracle_layer_fp8
    _chk(fn(_p(x), T, d, N, M, Kp, S, I, _DT[dtype], _p(wr), _p(b),
            _p(a["w_gate"]), _p(a["w_gate_scale"]), _p(a["w_up"]), _p(a["w_up_scale"]),
            _p(a["w_down"]), _p(a["w_down_scale"]), _p(a["s_gate"]), _p(a["s_gate_scale"]),
            _p(a["s_up"]), _p(a["s_up_scale"]), _p(a["s_down"]), _p(a["s_down_scale"]),
            _p(toks), n, _p(y), _p(idx), _p(w), _p(mg)), "layer_w8a8" if _act8 else "layer_fp8")
    return y, idx, w, mg
