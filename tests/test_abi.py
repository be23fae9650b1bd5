"""The C-ABI library loads and exports every symbol include/moge.h declares;
host-side argument checks reject bad calls before any device work (no GPU needed)."""
import ctypes
import os
import re
import subprocess

import pytest
import torch

import mixture_grouped_experts_b200 as mg
from mixture_grouped_experts_b200 import build as mbuild

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "moge.h")


@pytest.fixture(scope="module")
def L():
    mbuild.build()
    return mg.lib()


def declared_symbols():
    txt = open(HEADER).read()
    return sorted(set(re.findall(r"MOGE_API\s+[\w\s\*]*?\b(moge_\w+)\s*\(", txt)))


def test_header_declares_the_boundary():
    names = declared_symbols()
    for n in ("moge_route", "moge_permute", "moge_grouped_ffn", "moge_combine", "moge_layer_forward"):
        assert n in names
    assert set(names) == set(mg.EXPORTS)


def test_boundary_calls_cite_their_passage():
    """Each piecewise call of the boundary states, in its own comment, the
    page and section that define its operation."""
    txt = open(HEADER).read()
    pages = ("techwalker", "reportify", "mokono", "hwcomputing")
    for name in ("moge_route", "moge_permute", "moge_grouped_ffn", "moge_shared_ffn",
                 "moge_combine"):
        decl = re.search(r"MOGE_API\s+int\s+%s\s*\(" % name, txt)
        assert decl, name
        comment = txt[:decl.start()].rsplit("/*", 1)[1]
        assert any(p in comment for p in pages) and "section" in comment, name


def test_library_exports_every_declared_symbol(L):
    out = subprocess.check_output(["nm", "-D", "--defined-only", mg.LIB_PATH], text=True)
    exported = {line.split()[-1] for line in out.splitlines() if " T " in line}
    for n in declared_symbols():
        assert n in exported, n
        assert getattr(L, n) is not None
    # nothing else leaks out of the library under the moge_ prefix
    assert {e for e in exported if e.startswith("moge_")} == set(declared_symbols())


def _shape(**kw):
    base = dict(T=64, d=256, N=16, M=4, Kp=1, S=1, I=128, dtype="f32")
    base.update(kw)
    return mg.LayerShape(**base)


def test_workspace_size_matches_layout(L):
    s = _shape()
    n = mg.workspace_size(s)
    K = s.M * s.Kp
    big = s.T * K * s.d * 4 + s.T * (K + s.S) * (s.I + s.d) * 4
    assert big < n < big + 64 * 1024
    b = mg.workspace_size(_shape(dtype="bf16"))
    assert b < n                                   # bf16 rows take half the bytes
    assert mg.workspace_size(_shape(T=0)) > 0


def test_w8a8_workspace_is_the_forward_workspace_plus_its_regions(L):
    """The W8A8 workspace: the forward workspace, then x's codes [T][d] bytes,
    the token scales [T] and [T*K] fp32, h in fp32 [T(K+S)][I], its row amax
    words and row scales [T(K+S)], every region 256-byte aligned (at least
    one 256-byte slot each, even when empty)."""
    a256 = lambda n: (max(n, 1) + 255) // 256 * 256
    for kw in (dict(), dict(T=1), dict(T=0), dict(T=456, d=5120, N=64, M=8, S=4, I=1344),
               dict(Kp=2, S=0, I=336, d=528)):
        s = _shape(dtype="bf16", **kw)
        K, hrows = s.M * s.Kp, s.T * (s.M * s.Kp + s.S)
        want = (mg.workspace_size(s) + a256(s.T * s.d) + a256(s.T * 4) + a256(s.T * K * 4)
                + a256(hrows * s.I * 4) + 2 * a256(hrows * 4))
        assert mg.w8a8_workspace_size(s) == want, kw


@pytest.mark.parametrize("kw,code", [
    (dict(N=15), mg.ERR_UNSUPPORTED),               # N % M != 0
    (dict(Kp=5), mg.ERR_UNSUPPORTED),               # Kp > N/M
    (dict(d=100), mg.ERR_UNSUPPORTED),              # d % 8 != 0
    (dict(I=12), mg.ERR_UNSUPPORTED),               # I % 8 != 0
    (dict(N=512, M=4), mg.ERR_UNSUPPORTED),         # N > 256
    (dict(T=-1), mg.ERR_INVALID_ARG),
    (dict(M=0), mg.ERR_INVALID_ARG),
    (dict(N=12, M=4, dtype="bf16"), mg.ERR_UNSUPPORTED),  # bf16 router needs N % 8 == 0
])
def test_invalid_configs_rejected_on_host(L, kw, code):
    s = _shape(**kw)
    assert L.moge_workspace_size(ctypes.byref(mg._cfg(s))) == 0
    rc = L.moge_route(ctypes.byref(mg._cfg(s)), *([None] * 11))
    assert rc == code
    assert len(L.moge_last_error()) > 0


def test_null_and_misaligned_pointers_rejected(L):
    s = _shape()
    c = ctypes.byref(mg._cfg(s))
    assert L.moge_layer_forward(c, *([None] * 13)) == mg.ERR_INVALID_ARG
    assert b"x" in L.moge_last_error()
    # misaligned (odd) pointers are refused before anything is enqueued
    rc = L.moge_permute(c, 0x1001, 0x2000, 0x3000, None)
    assert rc == mg.ERR_UNSUPPORTED and b"aligned" in L.moge_last_error()
    rc = L.moge_rmsnorm(c, 0x1000, ctypes.c_float(-1.0), 0x2000, None)
    assert rc == mg.ERR_INVALID_ARG


def test_no_cpu_fallback_when_library_missing(monkeypatch):
    monkeypatch.setattr(mg, "_lib", None)
    monkeypatch.setattr(mg, "LIB_PATH", "/nonexistent/libmoge.so")
    with pytest.raises(ImportError):
        mg.lib()


def test_fp8_entry_points_validate_on_host(L):
    # quantiser: shape and alignment rules before anything is enqueued
    assert L.moge_quantize_fp8_rows(0x1000, 4, 12, 0x2000, 0x3000, None) == mg.ERR_UNSUPPORTED
    assert b"multiple of 8" in L.moge_last_error()
    assert L.moge_quantize_fp8_rows(0x1000, 4, 16, 0x2004, 0x3000, None) == mg.ERR_UNSUPPORTED
    assert L.moge_quantize_fp8_rows(None, 4, 16, 0x2000, 0x3000, None) == mg.ERR_INVALID_ARG
    assert L.moge_quantize_fp8_rows(None, 0, 16, None, None, None) == mg.OK
    # layer: bf16 only, 16-byte rows of codes, both sides' pointers present
    f8 = mg.moge_fp8_experts(0x1000, 0x2000, 0x3000, 0x4000, 0x5000, 0x6000)
    args = (0x7000, 0x8000, None, ctypes.byref(f8), ctypes.byref(f8), None, 0x9000, 0xA000, None)
    rc = L.moge_layer_forward_fp8(ctypes.byref(mg._cfg(_shape(dtype="f32"))), *args)
    assert rc == mg.ERR_UNSUPPORTED and b"BF16" in L.moge_last_error()
    rc = L.moge_layer_forward_fp8(ctypes.byref(mg._cfg(_shape(dtype="bf16", I=136))), *args)
    assert rc == mg.ERR_UNSUPPORTED and b"% 16" in L.moge_last_error()
    rc = L.moge_layer_forward_fp8(ctypes.byref(mg._cfg(_shape(dtype="bf16"))), 0x7000, 0x8000, None,
                                  None, ctypes.byref(f8), None, 0x9000, 0xA000, None)
    assert rc == mg.ERR_INVALID_ARG and b"routed" in L.moge_last_error()
    rc = L.moge_layer_forward_fp8(ctypes.byref(mg._cfg(_shape(dtype="bf16"))), 0x7000, 0x8000, None,
                                  ctypes.byref(f8), None, None, 0x9000, 0xA000, None)
    assert rc == mg.ERR_INVALID_ARG and b"shared" in L.moge_last_error()
    bad = mg.moge_fp8_experts(0x1000, 0x2000, 0x3000, 0x4002, 0x5000, 0x6000)
    rc = L.moge_layer_forward_fp8(ctypes.byref(mg._cfg(_shape(dtype="bf16"))), 0x7000, 0x8000, None,
                                  ctypes.byref(bad), ctypes.byref(f8), None, 0x9000, 0xA000, None)
    assert rc == mg.ERR_UNSUPPORTED and b"gate_scale" in L.moge_last_error()


def test_w8a8_entry_points_validate_on_host(L):
    s = _shape(dtype="bf16")
    K, hrows = s.M * s.Kp, s.T * (s.M * s.Kp + s.S)
    # the forward workspace, then x's codes, two scale arrays, h in fp32 and
    # its amax words and scales
    extra = s.T * s.d + s.T * 4 + s.T * K * 4 + hrows * s.I * 4 + 2 * hrows * 4
    n = mg.w8a8_workspace_size(s)
    assert mg.workspace_size(s) + extra <= n <= mg.workspace_size(s) + extra + 6 * 256
    assert L.moge_w8a8_workspace_size(ctypes.byref(mg._cfg(_shape(M=3)))) == 0
    f8 = mg.moge_fp8_experts(0x1000, 0x2000, 0x3000, 0x4000, 0x5000, 0x6000)
    args = (0x7000, 0x8000, None, ctypes.byref(f8), ctypes.byref(f8), None, 0x9000, 0xA000, None)
    rc = L.moge_layer_forward_w8a8(ctypes.byref(mg._cfg(_shape(dtype="f32"))), *args)
    assert rc == mg.ERR_UNSUPPORTED and b"BF16" in L.moge_last_error()
    rc = L.moge_layer_forward_w8a8(ctypes.byref(mg._cfg(_shape(dtype="bf16", d=264))), *args)
    assert rc == mg.ERR_UNSUPPORTED and b"% 16" in L.moge_last_error()
    rc = L.moge_layer_forward_w8a8(ctypes.byref(mg._cfg(s)), 0x7000, 0x8000, None, None,
                                   ctypes.byref(f8), None, 0x9000, 0xA000, None)
    assert rc == mg.ERR_INVALID_ARG and b"routed" in L.moge_last_error()
    rc = L.moge_layer_forward_w8a8(ctypes.byref(mg._cfg(s)), 0x7000, 0x8000, None,
                                   ctypes.byref(f8), ctypes.byref(f8), None, 0x7000, 0xA000, None)
    assert rc == mg.ERR_INVALID_ARG and b"alias" in L.moge_last_error()
    rc = L.moge_layer_forward_w8a8(ctypes.byref(mg._cfg(s)), 0x7000, 0x8000, None,
                                   ctypes.byref(f8), ctypes.byref(f8), None, 0x9000, None, None)
    assert rc == mg.ERR_INVALID_ARG and b"workspace" in L.moge_last_error()


def test_undersized_workspace_refused_before_the_call(L):
    # the C ABI cannot see a workspace's size; the binding checks torch ones
    s = _shape(dtype="bf16")
    small = torch.empty(mg.workspace_size(s), dtype=torch.uint8)   # the plain layer's size
    w8 = {k: None for k in mg.FP8_KEYS}
    with pytest.raises(mg.MogeError, match="moge_layer_forward_w8a8 needs"):
        mg.moge_layer_forward_w8a8(s, None, {}, w8, small)
    with pytest.raises(mg.MogeError, match="moge_layer_forward needs"):
        mg.moge_layer_forward(s, None, {}, small[:-1])
    with pytest.raises(mg.MogeError, match="moge_layer_backward needs"):
        mg.moge_layer_backward(s, None, {}, None, small)


def test_wait_selftest_validates_on_host(L):
    assert L.moge_selftest_waits(0, 0x1000, None) == mg.ERR_INVALID_ARG
    assert L.moge_selftest_waits(2000001, 0x1000, None) == mg.ERR_INVALID_ARG
    assert L.moge_selftest_waits(1000, None, None) == mg.ERR_INVALID_ARG
    assert L.moge_selftest_waits(1000, 0x1002, None) == mg.ERR_UNSUPPORTED


def test_expert_parallel_entry_points_validate_on_host(L):
    c = mg.moge_config(64, 256, 16, 4, 1, 1, 128, mg.MOGE_BF16)
    assert L.moge_ep_workspace_size(ctypes.byref(c), 4) > 0
    assert L.moge_ep_workspace_size(ctypes.byref(c), 3) == 0   # 3 does not divide M = 4
    assert L.moge_ep_workspace_size(ctypes.byref(c), 0) == 0
    args = [None] * 12
    assert L.moge_layer_forward_ep_local(ctypes.byref(c), 4, 4, *args) == mg.ERR_INVALID_ARG
    assert L.moge_layer_forward_ep_local(ctypes.byref(c), 0, 3, *args) == mg.ERR_UNSUPPORTED
    assert L.moge_layer_forward_ep_local(ctypes.byref(c), 0, 2, *args) == mg.ERR_INVALID_ARG  # y_part NULL
    assert L.moge_ep_finish(ctypes.byref(c), -1, None, None, None, None) == mg.ERR_INVALID_ARG
    assert L.moge_ep_finish(ctypes.byref(c), 4, 0x1008, None, 0x1000, None) == mg.ERR_UNSUPPORTED


def test_streaming_host_call_validates_on_host(L):
    c = mg.moge_config(64, 256, 16, 4, 1, 1, 128, mg.MOGE_BF16)
    args = [None] * 14
    assert L.moge_layer_forward_host_stream(ctypes.byref(c), -1, *args) == mg.ERR_INVALID_ARG
    assert L.moge_layer_forward_host_stream(ctypes.byref(c), 0, *args) == mg.OK  # nothing to do
    assert L.moge_layer_forward_host_stream(ctypes.byref(c), 2, *args) == mg.ERR_INVALID_ARG  # host NULL
    # x_host, w_router, bias, w_gate, w_up, w_down, s_gate, s_up, s_down, y_host,
    # x_dev2 (misaligned), y_dev2, workspace, stream
    bad = [0x1000] + [None] * 8 + [0x2000, 0x3008, 0x4000, None, None]
    assert L.moge_layer_forward_host_stream(ctypes.byref(c), 2, *bad) == mg.ERR_UNSUPPORTED
