"""Thin Python binding of libmoge.so, the B200 (sm_100a) MoGE layer: forward,
training forward + backward, and the expert-parallel local step.

Argument marshalling only: every step of the layer runs in the library's CUDA
kernels. PyTorch provides device memory and streams. The entry points carry
the names of the C ABI in include/moge.h; each takes torch tensors on the
current CUDA device (bf16 tensors for a bf16 layer, float32 for an fp32 one,
int32 indices, float32 scores) and enqueues on the current torch stream.

There is no fallback: if libmoge.so is missing or cannot be loaded, loading
it raises.
"""
from __future__ import annotations

import ctypes
import os
from dataclasses import dataclass
from typing import Optional

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libmoge.so")

MOGE_F32, MOGE_BF16 = 0, 1
OK, ERR_INVALID_ARG, ERR_UNSUPPORTED, ERR_CUDA, ERR_TIMEOUT, ERR_DEVICE = range(6)
_DT = {"f32": MOGE_F32, "bf16": MOGE_BF16}
_TORCH_DT = {"f32": torch.float32, "bf16": torch.bfloat16}

EXPORTS = ["moge_workspace_size", "moge_last_error", "moge_check_device_errors", "moge_route",
           "moge_permute", "moge_grouped_ffn", "moge_shared_ffn", "moge_combine",
           "moge_layer_forward", "moge_layer_forward_host", "moge_workspace_routing",
           "moge_rmsnorm", "moge_stage_timing", "moge_stage_times", "moge_route_noalloc",
           "moge_quantize_fp8_rows", "moge_layer_forward_fp8", "moge_selftest_waits",
           "moge_train_workspace_size", "moge_layer_forward_train", "moge_layer_backward",
           "moge_ep_workspace_size", "moge_layer_forward_ep_local", "moge_ep_finish",
           "moge_layer_forward_host_stream", "moge_w8a8_workspace_size", "moge_layer_forward_w8a8"]
STAGES = ("router", "scan", "permute", "ffn", "combine")


class MogeError(RuntimeError):
    def __init__(self, code: int, msg: str):
        super().__init__("moge error %d: %s" % (code, msg))
        self.code = code


class moge_config(ctypes.Structure):
    _fields_ = [(n, ctypes.c_int) for n in ("T", "d", "N", "M", "Kp", "S", "I", "dtype")]


class moge_fp8_experts(ctypes.Structure):
    _fields_ = [(n, ctypes.c_void_p) for n in ("gate", "up", "down", "gate_scale", "up_scale",
                                               "down_scale")]


@dataclass(frozen=True)
class LayerShape:
    """Sizes of one MoGE layer: T tokens, hidden d, N routed experts in M
    groups, Kp picked per group, S shared experts, SwiGLU intermediate I."""
    T: int
    d: int
    N: int
    M: int
    Kp: int
    S: int
    I: int
    dtype: str = "bf16"

    @property
    def K(self) -> int:
        return self.M * self.Kp


def shape_of(obj, **over) -> LayerShape:
    """LayerShape from any object with the fields T, d, N, M, Kp, S, I, dtype."""
    kw = {f: getattr(obj, f) for f in ("T", "d", "N", "M", "Kp", "S", "I", "dtype")}
    kw.update(over)
    return LayerShape(**kw)


_lib = None


def lib() -> ctypes.CDLL:
    """Load libmoge.so (raises when it is missing: there is no fallback path)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise ImportError("libmoge.so not built: run `python -m mixture_grouped_experts_b200.build`")
        L = ctypes.CDLL(LIB_PATH)
        vp, cp, i32 = ctypes.c_void_p, ctypes.POINTER(moge_config), ctypes.c_int
        L.moge_workspace_size.argtypes = [cp]
        L.moge_workspace_size.restype = ctypes.c_size_t
        L.moge_last_error.argtypes = []
        L.moge_last_error.restype = ctypes.c_char_p
        L.moge_check_device_errors.argtypes = [vp]
        L.moge_route.argtypes = [cp] + [vp] * 11
        L.moge_permute.argtypes = [cp, vp, vp, vp, vp]
        L.moge_grouped_ffn.argtypes = [cp] + [vp] * 8
        L.moge_shared_ffn.argtypes = [cp] + [vp] * 7
        L.moge_combine.argtypes = [cp] + [vp] * 7
        L.moge_layer_forward.argtypes = [cp] + [vp] * 13
        L.moge_layer_forward_host.argtypes = [cp] + [vp] * 14
        L.moge_workspace_routing.argtypes = [cp, vp] + [ctypes.POINTER(vp)] * 4
        L.moge_rmsnorm.argtypes = [cp, vp, ctypes.c_float, vp, vp]
        L.moge_stage_timing.argtypes = [i32]
        L.moge_route_noalloc.argtypes = [cp] + [vp] * 10
        L.moge_stage_times.argtypes = [ctypes.POINTER(ctypes.c_double), ctypes.POINTER(ctypes.c_int64)]
        L.moge_quantize_fp8_rows.argtypes = [vp, ctypes.c_int64, ctypes.c_int64, vp, vp, vp]
        L.moge_selftest_waits.argtypes = [ctypes.c_int64, vp, vp]
        fp = ctypes.POINTER(moge_fp8_experts)
        L.moge_layer_forward_fp8.argtypes = [cp, vp, vp, vp, fp, fp, vp, vp, vp, vp]
        L.moge_layer_forward_w8a8.argtypes = [cp, vp, vp, vp, fp, fp, vp, vp, vp, vp]
        L.moge_w8a8_workspace_size.argtypes = [cp]
        L.moge_w8a8_workspace_size.restype = ctypes.c_size_t
        L.moge_train_workspace_size.argtypes = [cp]
        L.moge_train_workspace_size.restype = ctypes.c_size_t
        L.moge_layer_forward_train.argtypes = [cp] + [vp] * 12
        L.moge_layer_backward.argtypes = [cp, ctypes.c_float] + [vp] * 21
        L.moge_ep_workspace_size.argtypes = [cp, i32]
        L.moge_ep_workspace_size.restype = ctypes.c_size_t
        L.moge_layer_forward_ep_local.argtypes = [cp, i32, i32] + [vp] * 12
        L.moge_ep_finish.argtypes = [cp, ctypes.c_int64, vp, vp, vp, vp]
        L.moge_layer_forward_host_stream.argtypes = [cp, ctypes.c_int64] + [vp] * 14
        for n in EXPORTS:
            if n not in ("moge_workspace_size", "moge_last_error", "moge_train_workspace_size",
                         "moge_ep_workspace_size", "moge_w8a8_workspace_size"):
                getattr(L, n).restype = i32
        _lib = L
    return _lib


def _cfg(s: LayerShape) -> moge_config:
    return moge_config(s.T, s.d, s.N, s.M, s.Kp, s.S, s.I, _DT[s.dtype])


def _p(t) -> Optional[int]:
    if t is None:
        return None
    if isinstance(t, int):
        return t
    if not t.is_contiguous():
        raise ValueError("tensors passed to libmoge must be contiguous")
    return t.data_ptr()


def _stream(stream) -> Optional[int]:
    if stream is None:
        stream = torch.cuda.current_stream()
    return stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream)


def _chk(rc: int):
    if rc != OK:
        raise MogeError(rc, lib().moge_last_error().decode())


def workspace_size(s: LayerShape) -> int:
    n = lib().moge_workspace_size(ctypes.byref(_cfg(s)))
    if n == 0:
        raise MogeError(ERR_INVALID_ARG, lib().moge_last_error().decode())
    return n


def alloc_workspace(s: LayerShape, device=None) -> torch.Tensor:
    return torch.empty(workspace_size(s), dtype=torch.uint8, device=device or "cuda")


def train_workspace_size(s: LayerShape) -> int:
    n = lib().moge_train_workspace_size(ctypes.byref(_cfg(s)))
    if n == 0:
        raise MogeError(ERR_UNSUPPORTED, lib().moge_last_error().decode())
    return n


def alloc_train_workspace(s: LayerShape, device=None) -> torch.Tensor:
    return torch.empty(train_workspace_size(s), dtype=torch.uint8, device=device or "cuda")


def check_device_errors(stream=None):
    _chk(lib().moge_check_device_errors(_stream(stream)))


def moge_route(s: LayerShape, x, w_router, logit_bias, workspace, stream=None):
    """-> (topk_idx [T][K] i32, topk_w [T][K] f32, counts [N], offsets [N+1], perm_src [T*K], perm_dst [T][K])"""
    dev = x.device
    T, K, N = s.T, s.K, s.N
    idx = torch.empty((T, K), dtype=torch.int32, device=dev)
    w = torch.empty((T, K), dtype=torch.float32, device=dev)
    counts = torch.empty(N, dtype=torch.int32, device=dev)
    offsets = torch.empty(N + 1, dtype=torch.int32, device=dev)
    ps = torch.empty(max(T * K, 1), dtype=torch.int32, device=dev)
    pd = torch.empty((T, K), dtype=torch.int32, device=dev)
    _chk(lib().moge_route(ctypes.byref(_cfg(s)), _p(x), _p(w_router), _p(logit_bias), _p(idx),
                          _p(w), _p(counts), _p(offsets), _p(ps), _p(pd), _p(workspace),
                          _stream(stream)))
    return idx, w, counts, offsets, ps[:T * K], pd


def moge_route_noalloc(s: LayerShape, x, w_router, logit_bias, stream=None):
    """moge_route with its scratch in the library's fixed device array (no
    workspace, nothing allocated by the library); same results."""
    dev = x.device
    T, K, N = s.T, s.K, s.N
    idx = torch.empty((T, K), dtype=torch.int32, device=dev)
    w = torch.empty((T, K), dtype=torch.float32, device=dev)
    counts = torch.empty(N, dtype=torch.int32, device=dev)
    offsets = torch.empty(N + 1, dtype=torch.int32, device=dev)
    ps = torch.empty(max(T * K, 1), dtype=torch.int32, device=dev)
    pd = torch.empty((T, K), dtype=torch.int32, device=dev)
    _chk(lib().moge_route_noalloc(ctypes.byref(_cfg(s)), _p(x), _p(w_router), _p(logit_bias),
                                  _p(idx), _p(w), _p(counts), _p(offsets), _p(ps), _p(pd),
                                  _stream(stream)))
    return idx, w, counts, offsets, ps[:T * K], pd


def moge_permute(s: LayerShape, x, perm_src, x_perm=None, stream=None):
    if x_perm is None:
        x_perm = torch.empty((s.T * s.K, s.d), dtype=x.dtype, device=x.device)
    _chk(lib().moge_permute(ctypes.byref(_cfg(s)), _p(x), _p(perm_src), _p(x_perm), _stream(stream)))
    return x_perm


def moge_grouped_ffn(s: LayerShape, x_perm, offsets, w_gate, w_up, w_down, workspace,
                     y_perm=None, stream=None):
    if y_perm is None:
        y_perm = torch.empty((s.T * s.K, s.d), dtype=x_perm.dtype, device=x_perm.device)
    _chk(lib().moge_grouped_ffn(ctypes.byref(_cfg(s)), _p(x_perm), _p(offsets), _p(w_gate),
                                _p(w_up), _p(w_down), _p(y_perm), _p(workspace), _stream(stream)))
    return y_perm


def moge_shared_ffn(s: LayerShape, x, s_gate, s_up, s_down, workspace, y_shared=None, stream=None):
    if y_shared is None:
        y_shared = torch.empty((s.T, s.d), dtype=x.dtype, device=x.device)
    _chk(lib().moge_shared_ffn(ctypes.byref(_cfg(s)), _p(x), _p(s_gate), _p(s_up), _p(s_down),
                               _p(y_shared), _p(workspace), _stream(stream)))
    return y_shared


def moge_combine(s: LayerShape, y_perm, topk_w, perm_dst, y_shared=None, residual=None, y=None,
                 stream=None):
    if y is None:
        y = torch.empty((s.T, s.d), dtype=y_perm.dtype, device=y_perm.device)
    _chk(lib().moge_combine(ctypes.byref(_cfg(s)), _p(y_perm), _p(topk_w), _p(perm_dst),
                            _p(y_shared), _p(residual), _p(y), _stream(stream)))
    return y


def _need_workspace(workspace, nbytes: int, what: str):
    """A torch workspace smaller than the call needs is refused on the host
    (the C ABI takes a bare pointer and cannot check its size)."""
    if isinstance(workspace, torch.Tensor) and workspace.numel() * workspace.element_size() < nbytes:
        raise MogeError(ERR_INVALID_ARG, "workspace of %d bytes, %s needs %d" % (
            workspace.numel() * workspace.element_size(), what, nbytes))


def moge_layer_forward(s: LayerShape, x, w: dict, workspace, residual=None, y=None, stream=None):
    """w: dict with w_router, logit_bias (or None), w_gate, w_up, w_down, s_gate, s_up, s_down."""
    _need_workspace(workspace, workspace_size(s), "moge_layer_forward")
    if y is None:
        y = torch.empty((s.T, s.d), dtype=x.dtype, device=x.device)
    _chk(lib().moge_layer_forward(ctypes.byref(_cfg(s)), _p(x), _p(w["w_router"]),
                                  _p(w.get("logit_bias")), _p(w["w_gate"]), _p(w["w_up"]),
                                  _p(w["w_down"]), _p(w.get("s_gate")), _p(w.get("s_up")),
                                  _p(w.get("s_down")), _p(residual), _p(y), _p(workspace),
                                  _stream(stream)))
    return y


def moge_layer_forward_train(s: LayerShape, x, w: dict, workspace, y=None, stream=None):
    """Forward that keeps what moge_layer_backward needs in `workspace` (a training workspace)."""
    _need_workspace(workspace, train_workspace_size(s), "moge_layer_forward_train")
    if y is None:
        y = torch.empty((s.T, s.d), dtype=x.dtype, device=x.device)
    _chk(lib().moge_layer_forward_train(ctypes.byref(_cfg(s)), _p(x), _p(w["w_router"]),
                                        _p(w.get("logit_bias")), _p(w["w_gate"]), _p(w["w_up"]),
                                        _p(w["w_down"]), _p(w.get("s_gate")), _p(w.get("s_up")),
                                        _p(w.get("s_down")), _p(y), _p(workspace),
                                        _stream(stream)))
    return y


GRAD_KEYS = ("w_router", "w_gate", "w_up", "w_down", "s_gate", "s_up", "s_down")


def moge_layer_backward(s: LayerShape, x, w: dict, dy, workspace, alpha: float = 0.0, grads=None,
                        dx=None, aux=None, stream=None):
    """Gradients for the preceding moge_layer_forward_train on the same workspace.
    Returns (dx, grads) with grads keyed like the weights (GRAD_KEYS); `aux` (a
    device float32 tensor of one element, optional) receives the balance loss."""
    _need_workspace(workspace, train_workspace_size(s), "moge_layer_backward")
    if dx is None:
        dx = torch.empty_like(x)
    if grads is None:
        grads = {k: torch.empty_like(w[k]) for k in GRAD_KEYS if w.get(k) is not None}
    _chk(lib().moge_layer_backward(ctypes.byref(_cfg(s)), float(alpha), _p(x), _p(w["w_router"]),
                                   _p(w.get("logit_bias")), _p(w["w_gate"]), _p(w["w_up"]),
                                   _p(w["w_down"]), _p(w.get("s_gate")), _p(w.get("s_up")),
                                   _p(w.get("s_down")), _p(dy), _p(dx),
                                   *[_p(grads.get(k)) for k in GRAD_KEYS], _p(aux),
                                   _p(workspace), _stream(stream)))
    return dx, grads


# ---------------------------------------------------------------- expert parallelism
def ep_workspace_size(s: LayerShape, world: int) -> int:
    n = lib().moge_ep_workspace_size(ctypes.byref(_cfg(s)), int(world))
    if n == 0:
        raise MogeError(ERR_UNSUPPORTED, lib().moge_last_error().decode())
    return n


def alloc_ep_workspace(s: LayerShape, world: int, device=None) -> torch.Tensor:
    return torch.empty(ep_workspace_size(s, world), dtype=torch.uint8, device=device or "cuda")


def ep_shard_weights(w: dict, rank: int, world: int) -> dict:
    """Rank `rank`'s expert-parallel share of a layer's weights (see moge.h):
    the routed experts of its groups (views of the full tensors, contiguous)
    and rows [r I/world, (r+1) I/world) of every shared expert's gate and up
    with the matching columns of its down projection (contiguous copies). The
    router is replicated."""
    N, I = w["w_gate"].shape[0], w["w_gate"].shape[1]
    if N % world or I % world:
        raise ValueError("world must divide the expert count and I")
    n_loc, i_s = N // world, I // world
    e0, i0 = rank * n_loc, rank * i_s
    out = {"w_router": w["w_router"], "logit_bias": w.get("logit_bias")}
    for k in ("w_gate", "w_up", "w_down"):
        out[k] = w[k][e0:e0 + n_loc]
    if w.get("s_gate") is not None:
        out["s_gate"] = w["s_gate"][:, i0:i0 + i_s].contiguous()
        out["s_up"] = w["s_up"][:, i0:i0 + i_s].contiguous()
        out["s_down"] = w["s_down"][:, :, i0:i0 + i_s].contiguous()
    return out


def moge_layer_forward_ep_local(s: LayerShape, rank: int, world: int, x_all, w_local: dict,
                                workspace, y_part=None, stream=None):
    """This rank's fp32 partial y [T][d] of the layer (s: the whole layer's shape)."""
    if y_part is None:
        y_part = torch.empty((s.T, s.d), dtype=torch.float32, device=x_all.device)
    _chk(lib().moge_layer_forward_ep_local(ctypes.byref(_cfg(s)), int(rank), int(world), _p(x_all),
                                           _p(w_local["w_router"]), _p(w_local.get("logit_bias")),
                                           _p(w_local["w_gate"]), _p(w_local["w_up"]),
                                           _p(w_local["w_down"]), _p(w_local.get("s_gate")),
                                           _p(w_local.get("s_up")), _p(w_local.get("s_down")),
                                           _p(y_part), _p(workspace), _stream(stream)))
    return y_part


def moge_ep_finish(s: LayerShape, y_sum, residual=None, y=None, stream=None):
    """y = y_sum (+ residual) in the layer dtype."""
    if y is None:
        y = torch.empty(y_sum.shape, dtype=_TORCH_DT[s.dtype], device=y_sum.device)
    _chk(lib().moge_ep_finish(ctypes.byref(_cfg(s)), int(y_sum.shape[0]), _p(y_sum), _p(residual),
                              _p(y), _stream(stream)))
    return y


def ep_chunk_bounds(rows: int, chunks: int):
    """Row ranges [a, b) of a rank's tokens, one per chunk of the pipelined
    expert-parallel step (as even as possible; every rank uses the same)."""
    chunks = max(1, min(int(chunks), rows)) if rows > 0 else 1
    out, a = [], 0
    for j in range(chunks):
        b = a + rows // chunks + (1 if j < rows % chunks else 0)
        out.append((a, b))
        a = b
    return out


def ep_default_chunks(rows: int) -> int:
    """Chunks of the pipelined step for `rows` tokens per rank: one for
    decode-sized batches (each chunk streams this rank's expert weights again,
    which only pays once the GEMMs are compute-bound), else about one per 256
    tokens, at most 4."""
    return 1 if rows < 512 else min(4, rows // 256)


def ep_pipeline(x_local, bounds, gather, local, reduce, finish, comm_stream=None):
    """The chunk schedule of the expert-parallel step, independent of the
    device: for every chunk j (rows bounds[j] of this rank's x_local), gather
    (all ranks' rows of the chunk) -> local (this rank's partial of those
    tokens) -> reduce (sum over ranks, this rank's rows) -> finish (into the
    output rows of the chunk). On CUDA, with comm_stream given, every gather is
    issued at once on comm_stream, chunk j's local step waits only for its own
    gather, and chunk j's reduce runs on comm_stream while chunk j + 1's local
    step runs, so the collectives overlap the GEMMs. Returns the finish
    results in chunk order."""
    import torch
    n = len(bounds)
    if comm_stream is None:
        outs = []
        for a, b in bounds:
            outs.append(finish(a, b, reduce(local(gather(x_local[a:b])))))
        return outs
    cur = torch.cuda.current_stream()
    comm_stream.wait_stream(cur)
    gathered, ev_g = [], []
    with torch.cuda.stream(comm_stream):
        for a, b in bounds:
            gathered.append(gather(x_local[a:b]))
            ev_g.append(comm_stream.record_event())
    reduced, ev_r = [None] * n, [None] * n
    for j, (a, b) in enumerate(bounds):
        cur.wait_event(ev_g[j])
        part = local(gathered[j])
        comm_stream.wait_stream(cur)
        with torch.cuda.stream(comm_stream):
            reduced[j] = reduce(part)
            ev_r[j] = comm_stream.record_event()
            part.record_stream(comm_stream)
        gathered[j].record_stream(cur)
    outs = []
    for j, (a, b) in enumerate(bounds):
        cur.wait_event(ev_r[j])
        reduced[j].record_stream(cur)
        outs.append(finish(a, b, reduced[j]))
    return outs


def moge_layer_forward_ep(s: LayerShape, x_local, w_local: dict, workspace=None, group=None,
                          residual=None, chunks=None, comm_stream=None):
    """One layer step under expert parallelism on the ranks of `group` (each
    with its own x_local [T/world][d]; s is the whole layer's shape, T = all
    ranks' tokens): all-gather x, this rank's partial, reduce-scatter of the
    partials (NCCL), finish. Returns this rank's y [T/world][d].

    The step is pipelined over `chunks` token chunks (default
    ep_default_chunks): the gathers run on a side stream (comm_stream, created
    when not given) and chunk j's reduce-scatter overlaps chunk j + 1's local
    GEMMs. workspace: an expert-parallel workspace for the largest chunk
    (alloc_ep_workspace of that chunk's shape), allocated here when None."""
    import torch.distributed as dist
    world, rank = dist.get_world_size(group), dist.get_rank(group)
    rows = x_local.shape[0]
    if rows * world != s.T:
        raise ValueError("x_local must hold T / world rows")
    bounds = ep_chunk_bounds(rows, ep_default_chunks(rows) if chunks is None else chunks)
    big = max(b - a for a, b in bounds)
    if workspace is None:
        workspace = alloc_ep_workspace(shape_of(s, T=big * world), world, x_local.device)
    elif workspace.numel() < ep_workspace_size(shape_of(s, T=big * world), world):
        raise ValueError("workspace smaller than the largest chunk needs")
    y = torch.empty((rows, s.d), dtype=_TORCH_DT[s.dtype], device=x_local.device)

    def gather(xc):
        xa = torch.empty((xc.shape[0] * world, s.d), dtype=xc.dtype, device=xc.device)
        dist.all_gather_into_tensor(xa, xc.contiguous(), group=group)
        return xa

    def local(xa):
        return moge_layer_forward_ep_local(shape_of(s, T=xa.shape[0]), rank, world, xa, w_local,
                                           workspace)

    def reduce(part):
        out = torch.empty((part.shape[0] // world, s.d), dtype=torch.float32, device=part.device)
        dist.reduce_scatter_tensor(out, part, group=group)
        return out

    def finish(a, b, ysum):
        res = None if residual is None else residual[a:b]
        return moge_ep_finish(shape_of(s, T=b - a), ysum, res, y[a:b])

    if comm_stream is None and len(bounds) > 1:
        comm_stream = torch.cuda.Stream(device=x_local.device)
    ep_pipeline(x_local, bounds, gather, local, reduce, finish,
                comm_stream if len(bounds) > 1 else None)
    return y


def moge_layer_forward_host(s: LayerShape, x_host, w: dict, workspace, y_host, x_dev, y_dev,
                            stream=None):
    """Host x in, host y out (pinned CPU tensors); returns after the stream is synchronised."""
    _chk(lib().moge_layer_forward_host(ctypes.byref(_cfg(s)), _p(x_host), _p(w["w_router"]),
                                       _p(w.get("logit_bias")), _p(w["w_gate"]), _p(w["w_up"]),
                                       _p(w["w_down"]), _p(w.get("s_gate")), _p(w.get("s_up")),
                                       _p(w.get("s_down")), _p(y_host), _p(x_dev), _p(y_dev),
                                       _p(workspace), _stream(stream)))
    return y_host


def moge_layer_forward_host_stream(s: LayerShape, x_host, w: dict, workspace, y_host, x_dev2,
                                   y_dev2, stream=None):
    """A run of independent batches from and to (pinned) host memory, copies
    overlapped with compute: x_host, y_host [n][T][d]; x_dev2, y_dev2 [2][T][d]
    device buffers. Returns after every output is in y_host."""
    _chk(lib().moge_layer_forward_host_stream(ctypes.byref(_cfg(s)), int(x_host.shape[0]),
                                              _p(x_host), _p(w["w_router"]), _p(w.get("logit_bias")),
                                              _p(w["w_gate"]), _p(w["w_up"]), _p(w["w_down"]),
                                              _p(w.get("s_gate")), _p(w.get("s_up")),
                                              _p(w.get("s_down")), _p(y_host), _p(x_dev2),
                                              _p(y_dev2), _p(workspace), _stream(stream)))
    return y_host


def moge_workspace_routing(s: LayerShape, workspace):
    """Views of the routing the last moge_layer_forward wrote into `workspace`:
    (topk_idx [T][K], topk_w [T][K], counts [N], offsets [N+1])."""
    ptrs = [ctypes.c_void_p() for _ in range(4)]
    _chk(lib().moge_workspace_routing(ctypes.byref(_cfg(s)), _p(workspace),
                                      *[ctypes.byref(p) for p in ptrs]))
    base = workspace.data_ptr()
    out = []
    for p, n, dt in zip(ptrs, (s.T * s.K, s.T * s.K, s.N, s.N + 1),
                        (torch.int32, torch.float32, torch.int32, torch.int32)):
        off = p.value - base
        out.append(workspace[off:off + 4 * n].view(dt))
    return out[0].view(s.T, s.K), out[1].view(s.T, s.K), out[2], out[3]


def moge_rmsnorm(s: LayerShape, x, eps: float = 1e-6, u=None, stream=None):
    if u is None:
        u = torch.empty_like(x)
    _chk(lib().moge_rmsnorm(ctypes.byref(_cfg(s)), _p(x), float(eps), _p(u), _stream(stream)))
    return u


def to_device(a, dtype: str, device="cuda") -> torch.Tensor:
    """Host array (uint16 bf16 bit patterns or float32) -> device tensor of the layer dtype."""
    import numpy as np
    if a is None:
        return None
    if dtype == "bf16" and a.dtype == np.uint16:
        return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).to(device).view(torch.bfloat16)
    return torch.from_numpy(np.ascontiguousarray(a)).to(device)


def weights_to_device(inp: dict, dtype: str, device="cuda") -> dict:
    """The weight dict of a layer (host arrays) moved to the device; logit_bias stays fp32."""
    out = {}
    for k in ("w_router", "w_gate", "w_up", "w_down", "s_gate", "s_up", "s_down"):
        out[k] = to_device(inp[k], dtype, device) if inp.get(k) is not None and inp[k].size else None
    lb = inp.get("logit_bias")
    out["logit_bias"] = None if lb is None else torch.from_numpy(lb).to(device)
    return out


def moge_stage_timing(enable: bool):
    """Start (reset) or stop the per-launch CUDA-event timing of moge_layer_forward."""
    _chk(lib().moge_stage_timing(1 if enable else 0))


def moge_stage_times():
    """-> ({stage: total ms}, timed calls) accumulated since moge_stage_timing(True)."""
    ms = (ctypes.c_double * len(STAGES))()
    n = ctypes.c_int64()
    _chk(lib().moge_stage_times(ms, ctypes.byref(n)))
    return {k: ms[i] for i, k in enumerate(STAGES)}, n.value


# ----------------------------------------------------------------------------- fp8 weights
FP8_KEYS = ("w_gate", "w_up", "w_down", "s_gate", "s_up", "s_down")


def moge_quantize_fp8_rows(w, stream=None):
    """Per-row E4M3 quantisation of a bf16 device tensor [..., cols] ->
    (codes uint8 of the same shape, fp32 scales of shape w.shape[:-1])."""
    if w.dtype != torch.bfloat16:
        raise TypeError("moge_quantize_fp8_rows takes a bf16 tensor")
    cols = w.shape[-1]
    rows = w.numel() // cols
    q = torch.empty(w.shape, dtype=torch.uint8, device=w.device)
    sc = torch.empty(w.shape[:-1], dtype=torch.float32, device=w.device)
    _chk(lib().moge_quantize_fp8_rows(_p(w), rows, cols, _p(q), _p(sc), _stream(stream)))
    return q, sc


def experts_to_fp8(w: dict, stream=None) -> dict:
    """FP8 codes and row scales of every expert matrix of a device weight dict
    (keys w_gate ... s_down, and the same keys + "_scale"); router weights and
    logit_bias are not touched."""
    out = {}
    for k in FP8_KEYS:
        if w.get(k) is not None:
            out[k], out[k + "_scale"] = moge_quantize_fp8_rows(w[k], stream)
        else:
            out[k] = out[k + "_scale"] = None
    return out


def _fp8_side(w8: dict, prefix: str):
    if w8.get(prefix + "_gate") is None:
        return None
    return moge_fp8_experts(*[_p(w8[prefix + n]) for n in ("_gate", "_up", "_down", "_gate_scale",
                                                            "_up_scale", "_down_scale")])


def moge_layer_forward_fp8(s: LayerShape, x, w: dict, w8: dict, workspace, residual=None, y=None,
                           stream=None):
    """Layer with FP8 expert weights w8 (experts_to_fp8 form); w gives w_router
    and logit_bias."""
    _need_workspace(workspace, workspace_size(s), "moge_layer_forward_fp8")
    if y is None:
        y = torch.empty((s.T, s.d), dtype=x.dtype, device=x.device)
    routed, shared = _fp8_side(w8, "w"), _fp8_side(w8, "s")
    _chk(lib().moge_layer_forward_fp8(ctypes.byref(_cfg(s)), _p(x), _p(w["w_router"]),
                                      _p(w.get("logit_bias")),
                                      ctypes.byref(routed) if routed is not None else None,
                                      ctypes.byref(shared) if shared is not None else None,
                                      _p(residual), _p(y), _p(workspace), _stream(stream)))
    return y


def w8a8_workspace_size(s: LayerShape) -> int:
    n = lib().moge_w8a8_workspace_size(ctypes.byref(_cfg(s)))
    if n == 0:
        raise MogeError(ERR_INVALID_ARG, "invalid layer config %r" % (s,))
    return n


def alloc_w8a8_workspace(s: LayerShape, device=None) -> torch.Tensor:
    return torch.empty(w8a8_workspace_size(s), dtype=torch.uint8, device=device or "cuda")


def moge_layer_forward_w8a8(s: LayerShape, x, w: dict, w8: dict, workspace, residual=None,
                            y=None, stream=None):
    """Layer in W8A8: FP8 expert weights w8 (experts_to_fp8 form) and
    activations quantised per token inside the call; w gives w_router and
    logit_bias; workspace of w8a8_workspace_size bytes."""
    _need_workspace(workspace, w8a8_workspace_size(s), "moge_layer_forward_w8a8")
    if y is None:
        y = torch.empty((s.T, s.d), dtype=x.dtype, device=x.device)
    routed, shared = _fp8_side(w8, "w"), _fp8_side(w8, "s")
    _chk(lib().moge_layer_forward_w8a8(ctypes.byref(_cfg(s)), _p(x), _p(w["w_router"]),
                                       _p(w.get("logit_bias")),
                                       ctypes.byref(routed) if routed is not None else None,
                                       ctypes.byref(shared) if shared is not None else None,
                                       _p(residual), _p(y), _p(workspace), _stream(stream)))
    return y


def moge_selftest_waits(limit_us: int, out, stream=None):
    """Run the bounded-wait check (see moge.h): out (device int32[3]) receives
    [1, 1, 0] once both waits gave up; the next check_device_errors reports
    the timeout."""
    _chk(lib().moge_selftest_waits(int(limit_us), _p(out), _stream(stream)))
    return out
