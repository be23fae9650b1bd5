#!/usr/bin/env python
"""Benchmark of the MoGE FFN layer forward on B200 (one JSON line on rank 0).

A step is one moge_layer_forward over one batch: router GEMM + global softmax +
per-group top-K', scan/permute, grouped SwiGLU up- and down-projection
(tcgen05), combine with the shared experts. Workload: the decode layer
(T=456 tokens, d=5120, 64 experts in 8 groups, K'=1, 4 shared experts,
intermediate 1344, bf16), synthetic seeded inputs. The 2.8 GB of expert
weights read per step exceed the 126 MB L2, so no L2 flush is needed.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl moge|reference]

N > 1 (torchrun): every rank runs its own batch with replicated weights, no
collective on the data path (weak scaling); time = max over ranks.
--impl reference times the CPU oracle (fp64, 1 thread) on a bounded sample.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402

import synth  # noqa: E402

METRIC = "MoGE layer tokens/s; % of HBM roofline (decode) / bf16 TC peak (prefill)"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
# The grouped FFN kernel a layer runs: the single-SM kernel below PAIR_ROWS
# routed rows (T * M * K'), the CTA-pair kernel from there on.
PAIR_ROWS = 8193
FFN_KERNEL = ("ffn_tc_kernel (grouped gate+up GEMM with SwiGLU epilogue and down GEMM, one "
              "persistent launch)")
# Nominal B200 figures, reported beside the measured denominators: HBM3e
# ~8 TB/s and 2.25 PFLOP/s dense bf16.
NOMINAL = {"hbm_gbs": 8000.0, "bf16_tflops": 2250.0}
# DRAM traffic of the dominant kernel comes from an ncu capture summarised
# under profiles/: a line "traffic-record: {json}" there names the kernel, the
# workload, the DRAM bytes of one launch (dram__bytes_read.sum +
# dram__bytes_write.sum) and a hash of the code (comments left out) of the
# CUDA sources the capture ran. The bench reports it only while the sources
# still hash the same (else null: the kernel changed since the counters were
# taken).
TRAFFIC_RECORDS = ("profiles/ffn_tc_decode.md", "profiles/ffn_tc_pair_prefill.md",
                   "profiles/ffn_tc_w8a8_decode.md")
FFN_PAIR_KERNEL = ("ffn_tc_pair_kernel (the same grouped FFN on CTA pairs, 2-SM tcgen05 MMA, "
                   "one persistent launch)")
FFN_W8A8_KERNEL = ("ffn_tc_kernel<W8> (the single-SM grouped FFN on 8-bit operands, tcgen05 "
                   "kind::f8f6f4, h quantised per token between the projections, one launch)")


def code_of(text):
    """C / CUDA source without its comments and with runs of white space
    collapsed: what the compiler sees, so that editing a comment does not
    change a source's hash. String and character literals are kept as they
    are (a // inside one is not a comment)."""
    out, i, n = [], 0, len(text)
    while i < n:
        c = text[i]
        if c in "\"'":
            j = i + 1
            while j < n and text[j] != c:
                j += 2 if text[j] == "\\" else 1
            out.append(text[i:j + 1])
            i = j + 1
        elif text.startswith("//", i):
            j = text.find("\n", i)
            i = n if j < 0 else j
        elif text.startswith("/*", i):
            j = text.find("*/", i + 2)
            out.append(" ")
            i = n if j < 0 else j + 2
        else:
            out.append(c)
            i += 1
    return " ".join("".join(out).split())


def source_sha16(files=None):
    """Hash of the code (comments left out, code_of) of CUDA sources of the
    library: the listed files of csrc/ (or all of csrc/*.cu, *.cuh, *.h and
    the ABI header when None), the key under which a traffic record is valid."""
    import glob
    import hashlib
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "mixture_grouped_experts_b200", "csrc")
    if files is None:
        paths = sorted(glob.glob(os.path.join(csrc, "*.cu")) + glob.glob(os.path.join(csrc, "*.cuh"))
                       + glob.glob(os.path.join(csrc, "*.h"))) + [os.path.join(ROOT, "include", "moge.h")]
    else:
        paths = [os.path.join(csrc, f) for f in files]
    for f in paths:
        h.update(os.path.basename(f).encode())
        h.update(code_of(open(f, encoding="utf-8").read()).encode())
    return h.hexdigest()[:16]


def traffic_record(kernel, workload):
    """(bytes per launch, source) of the committed ncu record for this kernel
    and workload when it was taken on the current sources of that kernel (the
    record's "files"), else (None, why)."""
    for rel in TRAFFIC_RECORDS:
        path = os.path.join(ROOT, rel)
        if not os.path.exists(path):
            continue
        for line in open(path):
            if not line.startswith("traffic-record:"):
                continue
            rec = json.loads(line.split(":", 1)[1])
            if rec.get("kernel") != kernel or rec.get("workload") != workload:
                continue
            sha = source_sha16(rec.get("files"))
            if rec.get("src_sha16") != sha:
                return None, "%s: captured on sources %s, now %s (kernel changed)" % (
                    rel, rec.get("src_sha16"), sha)
            return int(rec["dram_bytes_per_launch"]), "%s (ncu, sources %s)" % (rel, sha)
    return None, "no ncu record for %s on the %s workload" % (kernel, workload)


def layer_launches(cfg, fp8=False):
    """Kernel launches of one moge_layer_forward call, by the library's rules:
    router, scan, permute, grouped FFN, combine; bf16 layers of at most 8192
    routed rows (T * M * K') copy the permute inside the FFN launch."""
    if cfg.dtype == "bf16" and not fp8 and cfg.T * cfg.M * cfg.Kp <= 8192:
        return 4
    return 5


def host_cpu():
    """(logical CPUs, CPU model name) of this host."""
    model = ""
    try:
        for line in open("/proc/cpuinfo"):
            if line.startswith("model name"):
                model = line.split(":", 1)[1].strip()
                break
    except OSError:
        pass
    return os.cpu_count(), model


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return d, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


# ----------------------------------------------------------------------------- work model
def up_bytes(cfg, n_used):
    """Algorithmic bytes of one up-projection launch: gate+up weights of every
    expert that received a token, the B rows it reads (routed rows + x for the
    shared experts), and the h rows it writes; bf16."""
    T, d, I, K, S = cfg.T, cfg.d, cfg.I, cfg.K, cfg.S
    return 2 * ((n_used + S) * 2 * I * d + (T * K + T) * d + T * (K + S) * I)


def down_bytes(cfg, n_used):
    T, d, I, K, S = cfg.T, cfg.d, cfg.I, cfg.K, cfg.S
    return 2 * ((n_used + S) * d * I + T * (K + S) * I + T * (K + S) * d)


def up_flops(cfg):
    return 2.0 * (cfg.T * cfg.K + cfg.S * cfg.T) * cfg.d * 2 * cfg.I


def ffn_flops(cfg):
    """Both projections of every (token, expert) row: 2 * rows * d * 3I."""
    return 2.0 * (cfg.T * cfg.K + cfg.S * cfg.T) * cfg.d * 3 * cfg.I


def ffn_bytes(cfg, n_used):
    """Algorithmic bytes of the grouped-FFN launch (both projections)."""
    return up_bytes(cfg, n_used) + down_bytes(cfg, n_used)


def ffn_bytes_fp8(cfg, n_used):
    """Algorithmic bytes of the grouped-FFN launch with 8-bit weights: one byte
    per weight plus one fp32 scale per weight row, activations as in bf16."""
    T, d, I, K, S = cfg.T, cfg.d, cfg.I, cfg.K, cfg.S
    weights = (n_used + S) * (3 * I * d + 4 * (2 * I + d))
    acts = 2 * ((T * K + T) * d + 2 * T * (K + S) * I + T * (K + S) * d)
    return weights + acts


def layer_bytes_fp8(cfg, n_used):
    """Layer bytes with 8-bit expert weights (router stays bf16)."""
    return ((n_used + cfg.S) * (3 * cfg.I * cfg.d + 4 * (2 * cfg.I + cfg.d))
            + 2 * (cfg.N * cfg.d + 2 * cfg.T * cfg.d))


def layer_flops(cfg):
    return (cfg.T * cfg.K + cfg.S * cfg.T) * 6.0 * cfg.d * cfg.I + 2.0 * cfg.T * cfg.d * cfg.N


def train_flops(cfg):
    """FLOPs of one training step of the layer (moge_layer_forward_train +
    moge_layer_backward): the forward's, the backward's expert GEMMs (twice the
    forward FFN: dh and dx on the input side, dW_down and dW_gate / dW_up on
    the weight side) and the router's three (recomputed logits, dW_router, the
    router's share of dx)."""
    return layer_flops(cfg) + 2 * ffn_flops(cfg) + 3 * 2 * cfg.T * cfg.N * cfg.d


def layer_bytes(cfg, n_used):
    """Algorithmic bytes of the layer: each used expert's three matrices once,
    the router, x in and y out (no padding, no permute traffic)."""
    return 2 * ((n_used + cfg.S) * 3 * cfg.I * cfg.d + cfg.N * cfg.d + 2 * cfg.T * cfg.d)


# ----------------------------------------------------------------------------- clocks
class ClockSampler:
    Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index):
        self.idx = gpu_index
        self.proc = None
        self.path = None

    def start(self):
        try:
            fd, self.path = tempfile.mkstemp(suffix=".csv")
            os.close(fd)
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.idx), "--query-gpu=" + self.Q,
                 "--format=csv,noheader,nounits", "-lms", "200"],
                stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except (OSError, FileNotFoundError):
            self.proc = None

    def stop(self):
        if self.proc is None:
            return None
        time.sleep(0.25)
        self.proc.terminate()
        try:
            self.proc.wait(5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        rows = []
        for line in open(self.path):
            f = [x.strip() for x in line.split(",")]
            if len(f) < 9:
                continue
            try:
                rows.append((float(f[1]), float(f[2]), f[4:9]))
            except ValueError:
                continue
        os.unlink(self.path)
        if not rows:
            return None
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for _, _, r in rows for i in range(4) if r[i + 1] == "Active"})
        return {"sm_mhz": statistics.median(r[0] for r in rows), "sm_max_mhz": max(r[1] for r in rows),
                "reasons": reasons, "samples": len(rows)}


# ----------------------------------------------------------------------------- oracle legs
def oracle_sample(cfg, inp, tokens):
    """Time the CPU oracle on the listed tokens (full layer each)."""
    import oracle
    xd = oracle.to_double(inp["x"], cfg.dtype)
    t0 = time.perf_counter()
    oracle.layer(xd, inp, cfg.M, cfg.Kp, cfg.dtype, tokens=tokens)
    return time.perf_counter() - t0


def cpu_baseline(cfg, inp, n_tokens):
    toks = list(range(0, cfg.T, max(1, cfg.T // n_tokens)))[:n_tokens]
    dt = oracle_sample(cfg, inp, toks)
    nproc, model = host_cpu()
    return {"value": len(toks) / dt, "unit": "tokens/s", "cores": 1, "kind": "oracle",
            "nproc": nproc, "cpu_model": model,
            "sample": "%d of the %d tokens of the %s layer, full layer per token (routing over "
                      "%d experts, %d routed + %d shared SwiGLU experts), fp64 C, one thread; %.1f s"
                      % (len(toks), cfg.T, cfg.name, cfg.N, cfg.K, cfg.S, dt)}


def workload_config(cfg):
    return {"workload": "MoGE FFN layer forward, %s: T=%d tokens, d=%d, N=%d experts in M=%d groups, "
                        "K'=%d (K=%d), S=%d shared, SwiGLU I=%d, %s" % (
                            cfg.name, cfg.T, cfg.d, cfg.N, cfg.M, cfg.Kp, cfg.K, cfg.S, cfg.I, cfg.dtype),
            "T": cfg.T, "d": cfg.d, "N": cfg.N, "M": cfg.M, "Kp": cfg.Kp, "S": cfg.S, "I": cfg.I,
            "seed": cfg.seed,
            "l2": "inputs larger than L2: %.2f GB of expert weights read per step, no flush"
                  % (layer_bytes(cfg, cfg.N) / 1e9)}


def run_reference(args, cfg):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    inp = synth.layer_inputs(cfg)
    per_step = max(1, args.ref_tokens)
    rng = np.random.default_rng(0)
    for _ in range(args.warmup):
        oracle_sample(cfg, inp, rng.choice(cfg.T, per_step, replace=False).tolist())
    t = 0.0
    for _ in range(args.steps):
        t += oracle_sample(cfg, inp, rng.choice(cfg.T, per_step, replace=False).tolist())
    value = args.steps * per_step / t
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s",
            "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": 1000.0 * t / args.steps, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f64", "data": "synthetic (seeded normal inputs)",
            "config": dict(workload_config(cfg),
                           parallelism="replicas (dp%d), no collective" % args.gpus),
            "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": 1, "kind": "oracle",
                             "nproc": host_cpu()[0], "cpu_model": host_cpu()[1],
                             "sample": "each step: %d random tokens of the %d-token batch, full layer "
                                       "per token, fp64 C oracle, one thread" % (per_step, cfg.T)},
            "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


# ----------------------------------------------------------------------------- GPU arm
def measure(cfg, inp, steps, warmup, dist_on=False, with_e2e=True, fp8=False, w8a8=False):
    """Device-timed layer steps (+ per-launch stage times, + end-to-end through
    the host-buffer entry point). Returns a dict of raw measurements. With
    fp8 or w8a8, the expert weights are quantised on the device once (outside
    the timed region) and the layer runs moge_layer_forward_fp8 (weights-only
    8-bit) or moge_layer_forward_w8a8 (activations quantised inside the call)."""
    import torch
    import mixture_grouped_experts_b200 as mg

    s = mg.shape_of(cfg)
    x = mg.to_device(inp["x"], cfg.dtype)
    w = mg.weights_to_device(inp, cfg.dtype)
    ws = mg.alloc_w8a8_workspace(s) if w8a8 else mg.alloc_workspace(s)
    y = torch.empty_like(x)
    if fp8 or w8a8:
        w8 = mg.experts_to_fp8(w)
        torch.cuda.synchronize()
        for k in mg.FP8_KEYS:          # only the router stays in bf16
            w[k] = None
        torch.cuda.empty_cache()

        if w8a8:
            def fwd():
                mg.moge_layer_forward_w8a8(s, x, w, w8, ws, y=y)
        else:
            def fwd():
                mg.moge_layer_forward_fp8(s, x, w, w8, ws, y=y)
    else:
        def fwd():
            mg.moge_layer_forward(s, x, w, ws, y=y)
    for _ in range(max(warmup, 3)):
        fwd()
    torch.cuda.synchronize()
    mg.check_device_errors()
    counts = mg.moge_workspace_routing(s, ws)[2].cpu().numpy()
    n_used = int((counts > 0).sum())

    stream = torch.cuda.current_stream()
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    # timed region: the plain layer calls (no per-stage events between the
    # launches, which would break their programmatic overlap)
    if dist_on:
        torch.distributed.barrier()
    torch.cuda.synchronize()
    start.record(stream)
    for _ in range(steps):
        fwd()
    end.record(stream)
    torch.cuda.synchronize()
    if dist_on:
        torch.distributed.barrier()
    mg.check_device_errors()
    ms = start.elapsed_time(end) / steps
    # per-launch durations of the same workload, live, from the library's
    # CUDA-event stage timing (a separate loop of the same steps)
    mg.moge_stage_timing(True)
    for _ in range(steps):
        fwd()
    stage_ms, calls = mg.moge_stage_times()
    mg.moge_stage_timing(False)
    mg.check_device_errors()
    out = {"ms": ms, "stage_ms": {k: v / calls for k, v in stage_ms.items()}, "n_used": n_used,
           "counts": counts}
    if with_e2e and not (fp8 or w8a8):
        # end to end from pinned host memory: every step's x copied in and y
        # copied out inside the timed region. Headline: the streaming call (a
        # run of `steps` batches, copies overlapped with the neighbouring
        # batches' compute); also the one-batch synchronous call.
        xh = x.cpu().pin_memory()
        yh = torch.empty_like(xh).pin_memory()
        xd, yd = torch.empty_like(x), torch.empty_like(x)
        xs = xh.unsqueeze(0).repeat(steps, 1, 1).pin_memory()
        ys = torch.empty_like(xs).pin_memory()
        xd2 = torch.empty((2,) + tuple(x.shape), dtype=x.dtype, device=x.device)
        yd2 = torch.empty_like(xd2)
        mg.moge_layer_forward_host_stream(s, xs[:3], w, ws, ys[:3], xd2, yd2)
        for _ in range(3):
            mg.moge_layer_forward_host(s, xh, w, ws, yh, xd, yd)
        if dist_on:
            torch.distributed.barrier()
        torch.cuda.synchronize()
        start.record(stream)
        mg.moge_layer_forward_host_stream(s, xs, w, ws, ys, xd2, yd2)
        end.record(stream)
        torch.cuda.synchronize()
        out["e2e_ms"] = start.elapsed_time(end) / steps
        start.record(stream)
        for _ in range(steps):
            mg.moge_layer_forward_host(s, xh, w, ws, yh, xd, yd)
        end.record(stream)
        torch.cuda.synchronize()
        out["e2e_sync_ms"] = start.elapsed_time(end) / steps
        out["io_bytes"] = xh.numel() * xh.element_size()
    del x, w, ws, y
    if fp8 or w8a8:
        del w8
    torch.cuda.empty_cache()
    return out


def measure_train(cfg, inp, steps, warmup, alpha=0.01):
    """Device-timed training steps: forward (keeping what the backward needs)
    + backward with the balance loss; also the forward alone, same loop."""
    import torch
    import mixture_grouped_experts_b200 as mg

    s = mg.shape_of(cfg)
    x = mg.to_device(inp["x"], cfg.dtype)
    w = mg.weights_to_device(inp, cfg.dtype)
    dy = mg.to_device(synth.upstream_grad(cfg), "bf16")
    ws = mg.alloc_train_workspace(s)
    y = torch.empty_like(x)
    dx = torch.empty_like(x)
    grads = {k: torch.empty_like(w[k]) for k in mg.GRAD_KEYS if w.get(k) is not None}
    aux = torch.zeros(1, dtype=torch.float32, device="cuda")

    def fwd():
        mg.moge_layer_forward_train(s, x, w, ws, y=y)

    def step():
        fwd()
        mg.moge_layer_backward(s, x, w, dy, ws, alpha=alpha, grads=grads, dx=dx, aux=aux)

    stream = torch.cuda.current_stream()
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    out = {}
    for name, fn in (("step", step), ("fwd", fwd)):
        for _ in range(max(warmup, 3)):
            fn()
        torch.cuda.synchronize()
        start.record(stream)
        for _ in range(steps):
            fn()
        end.record(stream)
        torch.cuda.synchronize()
        out[name + "_ms"] = start.elapsed_time(end) / steps
    mg.check_device_errors()
    out["aux"] = float(aux.item())
    del x, w, dy, ws, y, dx, grads
    torch.cuda.empty_cache()
    return out


def measure_stack(cfg, steps, warmup):
    """Device-timed steps of the layer stack: for each of cfg.layers layers
    (independent weights), u = RMSNorm(x), x = x + layer(u). Weights are drawn
    on the device (seeded normal, std cfg.w_std): only timing depends on them;
    the stack's numerics are checked against the oracle by the tests."""
    import torch
    import mixture_grouped_experts_b200 as mg
    s = mg.shape_of(cfg)
    g = torch.Generator(device="cuda").manual_seed(cfg.seed)

    def rnd(*shape, std=cfg.w_std):
        return (torch.randn(shape, generator=g, device="cuda") * std).to(torch.bfloat16)

    E, I, d = cfg.N, cfg.I, cfg.d
    layers = []
    for _ in range(cfg.layers):
        layers.append({"w_router": rnd(E, d), "logit_bias": None, "w_gate": rnd(E, I, d),
                       "w_up": rnd(E, I, d), "w_down": rnd(E, d, I), "s_gate": rnd(cfg.S, I, d),
                       "s_up": rnd(cfg.S, I, d), "s_down": rnd(cfg.S, d, I)})
    x0 = rnd(cfg.T, d, std=cfg.x_std)
    xa, xb, u = torch.empty_like(x0), torch.empty_like(x0), torch.empty_like(x0)
    ws = mg.alloc_workspace(s)

    def step():
        cur, nxt = xa, xb
        cur.copy_(x0)
        for w in layers:
            mg.moge_rmsnorm(s, cur, 1e-6, u)
            mg.moge_layer_forward(s, u, w, ws, residual=cur, y=nxt)
            cur, nxt = nxt, cur

    for _ in range(max(warmup, 3)):
        step()
    torch.cuda.synchronize()
    mg.check_device_errors()
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    start.record()
    for _ in range(steps):
        step()
    end.record()
    torch.cuda.synchronize()
    mg.check_device_errors()
    ms = start.elapsed_time(end) / steps
    del layers, ws
    torch.cuda.empty_cache()
    return ms


def imbalance_score(counts, M, assignments):
    """Imbalance score of one batch: (busiest group's load - idlest group's
    load) / all (token, expert) assignments, the N experts in M contiguous
    groups."""
    import numpy as np
    loads = np.asarray(counts).reshape(M, -1).sum(axis=1)
    return {"score": float((loads.max() - loads.min()) / assignments),
            "group_loads": [int(v) for v in loads]}


def global_topk_imbalance(cfg, inp):
    """Route the same batch (same x, router weights and bias) by conventional
    global top-K (the library's router with one group of all N experts and K
    picks) and report its imbalance score over the layer's M groups."""
    import torch
    import mixture_grouped_experts_b200 as mg
    s1 = mg.shape_of(cfg, M=1, Kp=cfg.K, S=0)
    x = mg.to_device(inp["x"], cfg.dtype)
    wr = mg.to_device(inp["w_router"], cfg.dtype)
    lb = inp.get("logit_bias")
    lb = None if lb is None else torch.from_numpy(lb).cuda()
    ws = mg.alloc_workspace(s1)
    counts = mg.moge_route(s1, x, wr, lb, ws)[2]
    torch.cuda.synchronize()
    mg.check_device_errors()
    out = imbalance_score(counts.cpu().numpy(), cfg.M, cfg.T * cfg.K)
    out["routing"] = "global top-%d of %d experts on the same logits (library router, M=1)" % (
        cfg.K, cfg.N)
    del x, wr, ws
    torch.cuda.empty_cache()
    return out


def max_over_ranks(v, dist_on):
    """Max of a per-rank scalar over all ranks (identity on one process).
    Uses a CUDA tensor under NCCL and a CPU tensor under gloo."""
    if not dist_on:
        return v
    import torch
    dev = "cuda" if torch.distributed.get_backend() == "nccl" else "cpu"
    t = torch.tensor([v], dtype=torch.float64, device=dev)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return float(t.item())


def rank_inputs(cfg, rank, with_weights=True):
    """Inputs of one data-parallel rank: every rank holds the same weights
    (replicas) and its own token batch (x drawn from a rank-specific stream)."""
    inp = synth.layer_inputs(cfg, x_stream_offset=rank) if with_weights else {
        "x": synth.normal(cfg.seed, synth.STREAM_X + 1000 * rank, cfg.T * cfg.d, cfg.x_std,
                          cfg.dtype).reshape(cfg.T, cfg.d)}
    return inp


def ep_rank_bytes(cfg, world):
    """Expert-weight bytes one rank streams per expert-parallel step: its N/world
    routed experts and an I/world slice of every shared expert."""
    return (cfg.N // world + cfg.S / world) * 3 * cfg.I * cfg.d * 2


def run_ep(args, cfg, world, rank, local, dist_on, peaks):
    """--ep: the layer under expert parallelism (strong scaling: the workload's
    T tokens split over the ranks; each rank holds N/world experts and an
    I/world slice of the shared ones; all-gather + reduce-scatter over NCCL)."""
    import socket
    import torch
    import torch.distributed as dist
    import mixture_grouped_experts_b200 as mg
    if not dist_on:  # one rank: a world-1 NCCL group, so that the same driver runs
        sk = socket.socket()
        sk.bind(("127.0.0.1", 0))
        port = sk.getsockname()[1]
        sk.close()
        dist.init_process_group("nccl", init_method="tcp://127.0.0.1:%d" % port, rank=0,
                                world_size=1)
    if cfg.T % world or cfg.M % world or cfg.I % world:
        raise SystemExit("--ep needs world to divide T, M and I")
    s = mg.shape_of(cfg)
    inp = synth.layer_inputs(cfg)
    rows = cfg.T // world
    x = mg.to_device(inp["x"][rank * rows:(rank + 1) * rows], cfg.dtype)
    w = mg.weights_to_device(inp, cfg.dtype)
    wl = mg.ep_shard_weights(w, rank, world)
    wl = {k: (v.clone() if torch.is_tensor(v) else v) for k, v in wl.items()}
    del w, inp
    torch.cuda.empty_cache()
    ws = mg.alloc_ep_workspace(s, world)

    chunks = len(mg.ep_chunk_bounds(rows, mg.ep_default_chunks(rows)))
    comm = torch.cuda.Stream()

    def step():
        return mg.moge_layer_forward_ep(s, x, wl, ws, comm_stream=comm)

    for _ in range(max(args.warmup, 3)):
        step()
    torch.cuda.synchronize()
    mg.check_device_errors()
    sampler = ClockSampler(local)
    sampler.start()
    stream = torch.cuda.current_stream()
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    dist.barrier()
    torch.cuda.synchronize()
    start.record(stream)
    for _ in range(args.steps):
        step()
    end.record(stream)
    torch.cuda.synchronize()
    dist.barrier()
    clocks = sampler.stop()
    mg.check_device_errors()
    ms = max_over_ranks(start.elapsed_time(end) / args.steps, True)
    hbm = peaks["hbm_gbs"]
    rb = ep_rank_bytes(cfg, world)
    line = {"metric": METRIC, "value": cfg.T / (ms / 1e3), "unit": "tokens/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True,
            "scaling": "strong", "vs_baseline": None, "dtype": "bf16",
            "data": "synthetic (seeded normal inputs, random-init weights)",
            "config": dict(workload_config(cfg),
                           parallelism="ep%d: groups %d per rank, shared experts split by "
                                       "features, all-gather + reduce-scatter (NCCL) pipelined "
                                       "over %d token chunk(s) on a side stream"
                                       % (world, cfg.M // world, chunks)),
            "roofline": {"bound": "hbm", "kernel": "whole expert-parallel step (per rank)",
                         "achieved": rb / (ms / 1e3) / 1e9, "peak": hbm, "unit": "GB/s",
                         "frac": rb / (ms / 1e3) / 1e9 / hbm,
                         "algorithmic_bytes_per_rank": rb, "traffic": None},
            "e2e": None,
            # per chunk: router, localize, scan, permute, grouped FFN, combine,
            # (plan + shared-slice FFN), finish; NCCL's kernels not counted
            "gpu_launches": chunks * (7 + (2 if cfg.S else 0)) * args.steps,
            "clocks": clocks}
    if rank == 0:
        print(json.dumps(line), flush=True)
    dist.destroy_process_group()


def job_throughput(tokens_per_rank, world, max_ms):
    """Whole-job tokens/s: all ranks' tokens over the slowest rank's step time."""
    return world * tokens_per_rank / (max_ms / 1e3)


def arg_parser() -> argparse.ArgumentParser:
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="moge", choices=["moge", "reference"])
    ap.add_argument("--config", default="decode", choices=["decode", "prefill", "skew"])
    ap.add_argument("--no-secondary", action="store_true", help="skip the prefill side measurement")
    ap.add_argument("--cpu-tokens", type=int, default=16, help="tokens in the CPU-baseline sample (0: skip)")
    ap.add_argument("--no-e2e", action="store_true", help="skip the host-buffer end-to-end leg")
    ap.add_argument("--no-fp8", action="store_true",
                    help="skip the 8-bit side measurements (weights-only and W8A8)")
    ap.add_argument("--arith", default="bf16", choices=["bf16", "w8a8"],
                    help="arithmetic of the main line: the bf16 layer, or the W8A8 layer "
                         "(8-bit weights and per-token 8-bit activations; no host-buffer leg)")
    ap.add_argument("--no-train", action="store_true", help="skip the training-step side measurement")
    ap.add_argument("--no-extra", action="store_true",
                    help="skip the skewed-router and 12-layer-stack side measurements")
    ap.add_argument("--ref-tokens", type=int, default=2, help="tokens per step of --impl reference")
    ap.add_argument("--ep", action="store_true",
                    help="expert parallelism over the ranks instead of independent replicas")
    return ap


def main():
    args = arg_parser().parse_args()
    cfg = synth.CONFIGS[args.config]
    if args.impl == "reference":
        run_reference(args, cfg)
        return

    import torch
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    dist_on = world > 1
    if dist_on:
        import datetime
        torch.cuda.set_device(local)
        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=300),
                                             device_id=torch.device("cuda", local))
    else:
        torch.cuda.set_device(0)
    import mixture_grouped_experts_b200 as mg
    mg.lib()
    peaks, peak_kind = load_peaks()
    if args.ep:
        run_ep(args, cfg, world, rank, local, dist_on, peaks)
        return

    inp = rank_inputs(cfg, rank)
    sampler = ClockSampler(local)
    sampler.start()
    w8 = args.arith == "w8a8"
    m = measure(cfg, inp, args.steps, args.warmup, dist_on, with_e2e=not (args.no_e2e or w8),
                w8a8=w8)
    clocks = sampler.stop()
    ms = max_over_ranks(m["ms"], dist_on)
    e2e_ms = max_over_ranks(m.get("e2e_ms", float("nan")), dist_on)
    n = world
    value = job_throughput(cfg.T, n, ms)

    su = m["stage_ms"]
    hbm = peaks["hbm_gbs"]
    tf_burst = peaks.get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"])
    tf_sust = peaks.get("bf16_tflops_sustained", FALLBACK_PEAKS["bf16_tflops_sustained"])
    lb = layer_bytes_fp8(cfg, m["n_used"]) if w8 else layer_bytes(cfg, m["n_used"])
    if w8:
        # the W8A8 grouped FFN: the layer's 8-bit algorithmic bytes over its live
        # time (HBM-bound at decode), or its flops against the 8-bit dense rate
        # (twice the measured bf16 burst peak, the nominal fp8 / bf16 ratio)
        traffic, tsrc = traffic_record("ffn_tc_kernel<W8>", cfg.name)
        if cfg.T * cfg.M * cfg.Kp < PAIR_ROWS:
            ach = lb / (su["ffn"] / 1e3) / 1e9
            roofline = {"bound": "hbm", "kernel": FFN_W8A8_KERNEL, "achieved": ach, "peak": hbm,
                        "unit": "GB/s", "frac": ach / hbm,
                        "peak_source": "%s hbm_gbs" % peak_kind,
                        "algorithmic_bytes_per_launch": lb,
                        "algorithmic_bytes_are": "used experts' 8-bit matrices and row scales "
                                                 "once + router + x in + y out",
                        "traffic": traffic, "traffic_source": tsrc, "kernel_ms": su["ffn"]}
        else:
            ftf = ffn_flops(cfg) / (su["ffn"] / 1e3) / 1e12
            roofline = {"bound": "tensor", "kernel": FFN_W8A8_KERNEL, "achieved": ftf,
                        "peak": 2 * tf_burst, "unit": "TFLOP/s", "frac": ftf / (2 * tf_burst),
                        "peak_source": "2 x %s bf16_tflops (burst): the nominal fp8/bf16 ratio"
                                       % peak_kind,
                        "algorithmic_flops_per_launch": ffn_flops(cfg),
                        "traffic": traffic, "traffic_source": tsrc, "kernel_ms": su["ffn"]}
    elif cfg.T * cfg.M * cfg.Kp < PAIR_ROWS:
        # algorithmic bytes of the layer (the used experts' three matrices once,
        # the router, x in, y out: no padding, permute or intermediate rows) over
        # the grouped FFN's live launch time
        ach = lb / (su["ffn"] / 1e3) / 1e9
        fb_incl = ffn_bytes(cfg, m["n_used"])
        traffic, tsrc = traffic_record("ffn_tc_kernel", cfg.name)
        roofline = {"bound": "hbm", "kernel": FFN_KERNEL,
                    "achieved": ach, "peak": hbm, "unit": "GB/s", "frac": ach / hbm,
                    "peak_source": "measured (MEASURED_PEAKS.json hbm_gbs)" if peak_kind == "measured"
                    else "fallback 6650 GB/s",
                    "traffic": traffic, "traffic_source": tsrc,
                    "nominal": {"peak": NOMINAL["hbm_gbs"], "unit": "GB/s",
                                "frac": ach / NOMINAL["hbm_gbs"]},
                    "algorithmic_bytes_per_launch": lb,
                    "algorithmic_bytes_are": "used experts' three matrices once + router + x in + y out",
                    "bytes_incl_intermediates": fb_incl,
                    "frac_incl_intermediates": fb_incl / (su["ffn"] / 1e3) / 1e9 / hbm,
                    "kernel_ms": su["ffn"]}
    else:  # prefill-sized batches: the contraction bounds the pair kernel
        ftf = ffn_flops(cfg) / (su["ffn"] / 1e3) / 1e12
        traffic, tsrc = traffic_record("ffn_tc_pair_kernel", cfg.name)
        roofline = {"bound": "tensor", "kernel": FFN_PAIR_KERNEL, "achieved": ftf, "peak": tf_burst,
                    "unit": "TFLOP/s", "frac": ftf / tf_burst,
                    "peak_source": "%s bf16_tflops (burst)" % peak_kind,
                    "sustained": {"peak": tf_sust, "frac": ftf / tf_sust},
                    "traffic": traffic, "traffic_source": tsrc,
                    "nominal": {"peak": NOMINAL["bf16_tflops"], "unit": "TFLOP/s",
                                "frac": ftf / NOMINAL["bf16_tflops"]},
                    "algorithmic_flops_per_launch": ffn_flops(cfg), "kernel_ms": su["ffn"]}
    line = {"metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": n, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "bf16", "data": "synthetic (seeded normal inputs, random-init weights)",
            "config": dict(workload_config(cfg), parallelism="replicas (dp%d), no collective" % n),
            "roofline": roofline,
            "layer_roofline": {"bound": "hbm", "achieved": lb / (ms / 1e3) / 1e9, "peak": hbm,
                               "unit": "GB/s", "frac": lb / (ms / 1e3) / 1e9 / hbm,
                               "nominal": {"peak": NOMINAL["hbm_gbs"], "unit": "GB/s",
                                           "frac": lb / (ms / 1e3) / 1e9 / NOMINAL["hbm_gbs"]},
                               "algorithmic_bytes": lb},
            "stage_ms": su,
            "e2e": {"value": job_throughput(cfg.T, n, e2e_ms), "unit": "tokens/s",
                    "h2d_bytes_per_step": m.get("io_bytes"), "d2h_bytes_per_step": m.get("io_bytes"),
                    "api": "moge_layer_forward_host_stream (a run of `steps` batches from pinned "
                           "host memory, each batch's x copied in and y copied out, the copies "
                           "overlapped with the neighbouring batches' compute)",
                    "sync_per_step": {"value": job_throughput(cfg.T, n, max_over_ranks(
                        m.get("e2e_sync_ms", float("nan")), dist_on)), "unit": "tokens/s",
                        "api": "moge_layer_forward_host (one batch, synchronised per step)"}},
            "gpu_launches": layer_launches(cfg) * args.steps,
            "clocks": clocks}
    if w8:
        line["dtype"] = "e4m3 (W8A8: expert weights and activations; router bf16, fp32 accumulation)"
        line["e2e"] = {"value": None, "unit": "tokens/s", "h2d_bytes_per_step": None,
                       "d2h_bytes_per_step": None,
                       "note": "the host-buffer entry points run the bf16 layer; the W8A8 layer "
                               "is device-timed only"}
        line["gpu_launches"] = layer_launches(cfg, fp8=True) * args.steps
    if rank == 0 and n == 1 and args.cpu_tokens > 0:
        line["cpu_baseline"] = cpu_baseline(cfg, inp, args.cpu_tokens)
    del inp
    if rank == 0 and n == 1 and not args.no_secondary and args.config == "decode":
        pcfg = synth.CONFIGS["prefill"]
        pinp = synth.layer_inputs(pcfg)
        ps = ClockSampler(local)
        ps.start()
        pm = measure(pcfg, pinp, max(5, args.steps // 2), args.warmup, False, with_e2e=False)
        pclk = ps.stop()
        tf = peaks.get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"])
        tfs = peaks.get("bf16_tflops_sustained", FALLBACK_PEAKS["bf16_tflops_sustained"])
        ffn_tf = ffn_flops(pcfg) / (pm["stage_ms"]["ffn"] / 1e3) / 1e12
        lay_tf = layer_flops(pcfg) / (pm["ms"] / 1e3) / 1e12
        ptraffic, ptsrc = traffic_record("ffn_tc_pair_kernel", pcfg.name)
        line["prefill"] = {
            "workload": workload_config(pcfg)["workload"],
            "value": pcfg.T / (pm["ms"] / 1e3), "unit": "tokens/s", "ms_per_step": pm["ms"],
            "roofline": {"bound": "tensor", "kernel": FFN_PAIR_KERNEL, "achieved": ffn_tf,
                         "peak": tf, "unit": "TFLOP/s", "frac": ffn_tf / tf,
                         "peak_source": "%s bf16_tflops (burst)" % peak_kind,
                         "traffic": ptraffic, "traffic_source": ptsrc,
                         "nominal": {"peak": NOMINAL["bf16_tflops"], "unit": "TFLOP/s",
                                     "frac": ffn_tf / NOMINAL["bf16_tflops"]}},
            "layer_roofline": {"bound": "tensor", "achieved": lay_tf, "peak": tf, "unit": "TFLOP/s",
                               "frac": lay_tf / tf, "peak_source": "%s bf16_tflops (burst)" % peak_kind,
                               "sustained": {"peak": tfs, "frac": lay_tf / tfs},
                               "algorithmic_flops": layer_flops(pcfg)},
            "gpu_launches_per_step": layer_launches(pcfg),
            "stage_ms": pm["stage_ms"], "clocks": pclk}
    if rank == 0 and n == 1 and not args.no_fp8 and not w8 and args.config == "decode":
        finp = synth.layer_inputs(cfg)
        fs = ClockSampler(local)
        fs.start()
        fm = measure(cfg, finp, args.steps, args.warmup, False, with_e2e=False, fp8=True)
        fclk = fs.stop()
        del finp
        fb8 = ffn_bytes_fp8(cfg, fm["n_used"])
        ach8 = fb8 / (fm["stage_ms"]["ffn"] / 1e3) / 1e9
        lb8 = layer_bytes_fp8(cfg, fm["n_used"])
        line["decode_fp8"] = {
            "workload": workload_config(cfg)["workload"],
            "weights": "expert weights as OCP E4M3 codes + one fp32 scale per row (weights-only "
                       "8-bit; router, activations, h and y bf16); quantised on the device before "
                       "the timed region",
            "value": cfg.T / (fm["ms"] / 1e3), "unit": "tokens/s", "ms_per_step": fm["ms"],
            "roofline": {"bound": "hbm", "kernel": "ffn_fp8_kernel", "achieved": ach8, "peak": hbm,
                         "unit": "GB/s", "frac": ach8 / hbm, "algorithmic_bytes_per_launch": fb8,
                         "kernel_ms": fm["stage_ms"]["ffn"]},
            "layer_roofline": {"achieved": lb8 / (fm["ms"] / 1e3) / 1e9, "peak": hbm, "unit": "GB/s",
                               "frac": lb8 / (fm["ms"] / 1e3) / 1e9 / hbm, "algorithmic_bytes": lb8},
            "gpu_launches_per_step": layer_launches(cfg, fp8=True),
            "stage_ms": fm["stage_ms"], "clocks": fclk}
        # W8A8: the same 8-bit weights, x and h quantised per token inside the
        # call, both operands of every expert GEMM E4M3 on the 8-bit MMA
        ainp = synth.layer_inputs(cfg)
        as_ = ClockSampler(local)
        as_.start()
        am = measure(cfg, ainp, args.steps, args.warmup, False, with_e2e=False, w8a8=True)
        aclk = as_.stop()
        del ainp
        lba = layer_bytes_fp8(cfg, am["n_used"])
        ach_a = lba / (am["stage_ms"]["ffn"] / 1e3) / 1e9
        atraffic, atsrc = traffic_record("ffn_tc_kernel<W8>", cfg.name)
        line["decode_w8a8"] = {
            "workload": workload_config(cfg)["workload"],
            "weights": "expert weights as OCP E4M3 codes + one fp32 scale per row; x and h "
                       "quantised per token (E4M3, fp32 scale amax/448) inside the call; router "
                       "bf16, y bf16; weights quantised on the device before the timed region",
            "value": cfg.T / (am["ms"] / 1e3), "unit": "tokens/s", "ms_per_step": am["ms"],
            "vs_bf16_layer": ms / am["ms"] if n == 1 else None,
            "roofline": {"bound": "hbm", "kernel": FFN_W8A8_KERNEL, "achieved": ach_a, "peak": hbm,
                         "unit": "GB/s", "frac": ach_a / hbm, "algorithmic_bytes_per_launch": lba,
                         "algorithmic_bytes_are": "used experts' 8-bit matrices and row scales "
                                                  "once + router + x in + y out",
                         "traffic": atraffic, "traffic_source": atsrc,
                         "kernel_ms": am["stage_ms"]["ffn"]},
            "layer_roofline": {"achieved": lba / (am["ms"] / 1e3) / 1e9, "peak": hbm, "unit": "GB/s",
                               "frac": lba / (am["ms"] / 1e3) / 1e9 / hbm, "algorithmic_bytes": lba},
            "gpu_launches_per_step": layer_launches(cfg, fp8=True),
            "stage_ms": am["stage_ms"], "clocks": aclk}
    if rank == 0 and n == 1 and not args.no_train and args.config == "decode":
        tcfg = synth.CONFIGS["prefill"]
        tinp = synth.layer_inputs(tcfg)
        ts = ClockSampler(local)
        ts.start()
        tm = measure_train(tcfg, tinp, max(5, args.steps // 2), args.warmup)
        tclk = ts.stop()
        del tinp
        tf = peaks.get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"])
        tfs = peaks.get("bf16_tflops_sustained", FALLBACK_PEAKS["bf16_tflops_sustained"])
        ach = train_flops(tcfg) / (tm["step_ms"] / 1e3) / 1e12
        bwd_ms = tm["step_ms"] - tm["fwd_ms"]
        bwd_tf = (train_flops(tcfg) - layer_flops(tcfg)) / (bwd_ms / 1e3) / 1e12
        line["train_prefill"] = {
            "workload": workload_config(tcfg)["workload"],
            "step": "moge_layer_forward_train + moge_layer_backward (all weight and input "
                    "gradients, batch balance loss alpha = 0.01)",
            "value": tcfg.T / (tm["step_ms"] / 1e3), "unit": "tokens/s",
            "ms_per_step": tm["step_ms"], "forward_ms": tm["fwd_ms"], "backward_ms": bwd_ms,
            "roofline": {"bound": "tensor", "kernel": "training step (forward + backward GEMMs)",
                         "achieved": ach, "peak": tf, "unit": "TFLOP/s", "frac": ach / tf,
                         "flops_per_step": train_flops(tcfg),
                         "peak_source": "%s bf16_tflops (burst: the timed region is tens of "
                                        "milliseconds)" % peak_kind,
                         "sustained": {"peak": tfs, "frac": ach / tfs}},
            "backward_tflops": bwd_tf, "clocks": tclk}
    if rank == 0 and n == 1 and not args.no_extra and args.config == "decode":
        kcfg = synth.CONFIGS["skew"]
        kinp = synth.layer_inputs(kcfg)
        ks = ClockSampler(local)
        ks.start()
        km = measure(kcfg, kinp, 5, args.warmup, False, with_e2e=False)
        kclk = ks.stop()
        del kinp
        tf = peaks.get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"])
        tfs = peaks.get("bf16_tflops_sustained", FALLBACK_PEAKS["bf16_tflops_sustained"])
        k_tf = layer_flops(kcfg) / (km["ms"] / 1e3) / 1e12
        cnt = km["counts"]
        gim = global_topk_imbalance(kcfg, synth.layer_inputs(kcfg))
        line["skew"] = {
            "workload": workload_config(kcfg)["workload"],
            "value": kcfg.T / (km["ms"] / 1e3), "unit": "tokens/s", "ms_per_step": km["ms"],
            "roofline": {"bound": "tensor", "kernel": "whole layer", "achieved": k_tf, "peak": tf,
                         "unit": "TFLOP/s", "frac": k_tf / tf,
                         "peak_source": "%s bf16_tflops (burst)" % peak_kind,
                         "sustained": {"peak": tfs, "frac": k_tf / tfs},
                         "algorithmic_flops": layer_flops(kcfg)},
            "expert_rows": {"max": int(cnt.max()), "min": int(cnt.min())},
            "group_rows": [int(cnt[g * (kcfg.N // kcfg.M):(g + 1) * (kcfg.N // kcfg.M)].sum())
                           for g in range(kcfg.M)],
            "imbalance_moge": imbalance_score(cnt, kcfg.M, kcfg.T * kcfg.K),
            "imbalance_global_top8": gim,
            "gpu_launches_per_step": layer_launches(kcfg),
            "stage_ms": km["stage_ms"], "clocks": kclk}
        scfg = synth.CONFIGS["stack12"]
        ss = ClockSampler(local)
        ss.start()
        sms = measure_stack(scfg, 5, args.warmup)
        sclk = ss.stop()
        sb = scfg.layers * layer_bytes(scfg, scfg.N) / (sms / 1e3) / 1e9
        line["stack12"] = {
            "workload": "12-layer stack of MoGE FFN blocks with pre-RMSNorm (eps 1e-6) and "
                        "residual, decode: T=456, d=5120, per layer 64 experts / 8 groups / K'=1, "
                        "4 shared, I=1344, bf16, independent weights per layer (33.8 GB)",
            "value": scfg.T / (sms / 1e3), "unit": "tokens/s", "ms_per_step": sms,
            "roofline": {"bound": "hbm", "achieved": sb, "peak": hbm, "unit": "GB/s",
                         "frac": sb / hbm, "algorithmic_bytes": scfg.layers * layer_bytes(scfg, scfg.N)},
            "clocks": sclk}
    if rank == 0:
        print(json.dumps(line), flush=True)
    if dist_on:
        torch.distributed.destroy_process_group()


if __name__ == "__main__":
    main()
