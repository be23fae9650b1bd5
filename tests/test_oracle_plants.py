"""The oracle's pins against planted mistakes (no GPU). Each case copies
oracle.c, plants one plausible mistake in the copy (a dropped term, a wrong
sign or index, a misread of the routing rule), builds it, and runs the pin
suites (test_oracle*.py) on that build in a child pytest: at least one pin
must fail. A control case builds the unchanged source the same way and must
pass every pin, so a failure is due to the plant and not to the harness.

The builds go to _build/oracle_plants/ at the repository root (ignored by
git). Nothing here touches the CUDA path."""
import os
import subprocess
import sys
from concurrent.futures import ThreadPoolExecutor

import pytest

import oracle

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SRC = os.path.join(ROOT, "oracle", "oracle.c")
OUT = os.path.join(ROOT, "_build", "oracle_plants")
PIN_SUITES = ["tests/test_oracle.py", "tests/test_oracle_bwd.py", "tests/test_oracle_fp8.py",
              "tests/test_oracle_w8a8.py", "tests/test_oracle_ep.py"]

# name -> [(text in oracle.c, replacement, which occurrence (0-based))]
PLANTS = {
    # combine weights: 1 instead of the picked expert's score
    "unweighted_picks": [("w[(size_t)t * K + g * Kp + j] = pt[best];",
                          "w[(size_t)t * K + g * Kp + j] = 1.0;", 0)],
    # combine weight read at the wrong expert (the group's first)
    "weight_of_wrong_expert": [("w[(size_t)t * K + g * Kp + j] = pt[best];",
                                "w[(size_t)t * K + g * Kp + j] = pt[g * G];", 0)],
    # groups as strided sets of experts instead of contiguous blocks
    "strided_groups": [("for (int e = g * G; e < (g + 1) * G; ++e) {",
                        "for (int e = g; e < N; e += M) {", 0),
                       ("for (int e = g * G; e < (g + 1) * G; ++e)\n",
                        "for (int e = g; e < N; e += M)\n", 0)],
    # equal scores go to the higher expert index
    "ties_to_higher_index": [("if (best < 0 || v > bv) { best = e; bv = v; }  /* ties: lower",
                              "if (best < 0 || v >= bv) { best = e; bv = v; }  /* ties: lower", 0)],
    # router bias subtracted
    "bias_sign": [("l[e] = dot(xt, w, d) + (bias ? (double)bias[e] : 0.0);",
                   "l[e] = dot(xt, w, d) - (bias ? (double)bias[e] : 0.0);", 0)],
    # SwiGLU with the gate and up products swapped
    "silu_on_up": [("h[i] = (g / (1.0 + exp(-g))) * u;", "h[i] = (u / (1.0 + exp(-u))) * g;", 0)],
    # shared experts left out of the layer
    "shared_dropped": [("for (int s = 0; s < S && rc == 0; ++s) {\n"
                        "            rc = oracle_expert_ffn(xt, expert_ptr(s_gate, dtype, (size_t)s, per),",
                        "for (int s = 0; s < 0 && rc == 0; ++s) {\n"
                        "            rc = oracle_expert_ffn(xt, expert_ptr(s_gate, dtype, (size_t)s, per),",
                        0)],
    # backward: sign error in the SiLU derivative
    "silu_derivative_sign": [("s * (1.0 + g[i] * (1.0 - s))", "s * (1.0 - g[i] * (1.0 - s))", 0)],
    # backward: softmax Jacobian without its centring term
    "router_grad_uncentred": [("const double dl = pt[e] * (dp[e] - pdp);",
                               "const double dl = pt[e] * dp[e];", 0)],
    # backward: balance-loss gradient without the 1/T of P_i
    "aux_grad_scale": [("for (int e = 0; e < N; ++e) dp[e] = alpha * f[e] / T;",
                        "for (int e = 0; e < N; ++e) dp[e] = alpha * f[e];", 0)],
    # backward: W_down gradient without the combine weight
    "dw_down_unweighted": [("if (gd) gd[(size_t)o * I + i] += w * dyt[o] * h[i];",
                            "if (gd) gd[(size_t)o * I + i] += dyt[o] * h[i];", 0)],
    # router rows read with a wrong stride
    "router_row_stride": [("load_row(w_router, dtype, (size_t)e * d, d, w);",
                           "load_row(w_router, dtype, (size_t)e * (d - 1), d, w);", 0)],
    # routed experts' W_up pointer taken from W_gate (copy-paste slip)
    "up_from_gate": [("expert_ptr(w_up, dtype, e, per),", "expert_ptr(w_gate, dtype, e, per),", 0)],
    # 8-bit weights: E4M3 exponent bias 8 instead of 7
    "e4m3_bias": [("ldexp(1.0 + m / 8.0, e - 7)", "ldexp(1.0 + m / 8.0, e - 8)", 0)],
    # W8A8: h left unquantised before the down product
    "w8a8_h_unquantised": [("    quantize_act_inplace(h, I, codes);\n", "", 0)],
    # W8A8: x left unquantised before the gate and up products
    "w8a8_x_unquantised": [("    quantize_act_inplace(xq, d, codes);\n", "", 0)],
    # W8A8: activation scale amax / 224 (codes saturate)
    "w8a8_act_scale": [("volatile float s = amax > 0.0f ? amax / 448.0f : 1.0f;",
                        "volatile float s = amax > 0.0f ? amax / 224.0f : 1.0f;", 1)],
    # W8A8: the layer's routed experts evaluated without activation quantisation
    "w8a8_layer_weights_only": [("                      oracle_expert_ffn_w8a8);",
                                 "                      oracle_expert_ffn_fp8);", 0)],
    # expert-parallel partial: routed outputs not weighted by their scores
    "ep_partial_unweighted": [("            if (rc) break;\n"
                               "            for (int o = 0; o < d; ++o) yt[o] += w[k] * tmp[o];\n"
                               "        }\n"
                               "        for (int s = 0; s < S && rc == 0 && I_s > 0; ++s) {",
                               "            if (rc) break;\n"
                               "            for (int o = 0; o < d; ++o) yt[o] += tmp[o];\n"
                               "        }\n"
                               "        for (int s = 0; s < S && rc == 0 && I_s > 0; ++s) {", 0)],
}


def _plant(src: str, edits) -> str:
    for old, new, which in edits:
        pos = -1
        for _ in range(which + 1):
            pos = src.find(old, pos + 1)
            assert pos >= 0, "plant site not found: %r" % old
        src = src[:pos] + new + src[pos + len(old):]
    return src


def _run_pins(name: str, src: str) -> subprocess.CompletedProcess:
    os.makedirs(OUT, exist_ok=True)
    c_path = os.path.join(OUT, "oracle_%s.c" % name)
    with open(c_path, "w") as f:
        f.write(src)
    lib = oracle.compile_lib(c_path, os.path.join(OUT, "liboracle_%s.so" % name))
    env = dict(os.environ, ORACLE_LIB=lib)
    return subprocess.run([sys.executable, "-m", "pytest", "-x", "-q", "-m", "not gpu",
                           "-p", "no:cacheprovider"] + PIN_SUITES,
                          cwd=ROOT, env=env, capture_output=True, text=True, timeout=600)


@pytest.fixture(scope="module")
def results():
    """Every build's child pytest, run side by side (each is one process)."""
    with open(SRC) as f:
        src = f.read()
    jobs = {"control": src}
    for name, edits in PLANTS.items():
        jobs[name] = _plant(src, edits)
        assert jobs[name] != src, name
    with ThreadPoolExecutor(max_workers=min(8, os.cpu_count() or 1)) as ex:
        futs = {name: ex.submit(_run_pins, name, text) for name, text in jobs.items()}
        return {name: f.result() for name, f in futs.items()}


def test_control_build_passes_every_pin(results):
    r = results["control"]
    assert r.returncode == 0, r.stdout[-2000:]


@pytest.mark.parametrize("name", sorted(PLANTS))
def test_pins_catch_planted_mistake(results, name):
    r = results[name]
    assert r.returncode == 1 and " failed" in r.stdout, (name, r.returncode, r.stdout[-1500:])
