"""The profile summaries' commands (no GPU): each one runs committed files only,
with arguments the benchmark accepts, every ncu command leaves the clocks
alone, and every kernel filter names a kernel that the sources define."""
import glob
import os
import re
import shlex

import bench

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CSRC = os.path.join(ROOT, "mixture_grouped_experts_b200", "csrc")


def _commands(md_text):
    """Shell commands of the fenced blocks, backslash continuations joined."""
    out = []
    for block in re.findall(r"```[a-z]*\n(.*?)```", md_text, flags=re.S):
        joined = re.sub(r"\\\n\s*", " ", block)
        out += [ln.strip() for ln in joined.splitlines() if ln.strip()]
    return out


def _bench_args(cmd):
    """Argument lists given to bench.py in one command line (before any
    redirection or chaining)."""
    found = []
    for m in re.finditer(r"python bench\.py((?:\s+[^\s>&|;]+)*)", cmd):
        found.append(shlex.split(m.group(1)))
    return found


def _kernel_names():
    names = set()
    for path in glob.glob(os.path.join(CSRC, "*.cu")):
        src = open(path).read()
        names |= set(re.findall(r"__global__.{0,200}?\b(\w+_kernel)\s*\(", src, flags=re.S))
    return names


PROFILES = sorted(glob.glob(os.path.join(ROOT, "profiles", "*.md")))


def test_every_profile_has_a_command():
    assert PROFILES
    for path in PROFILES:
        cmds = _commands(open(path).read())
        assert any(_bench_args(c) for c in cmds), os.path.basename(path)


def test_profile_commands_parse_and_leave_clocks_alone():
    parser = bench.arg_parser()
    kernels = _kernel_names()
    assert {"ffn_tc_kernel", "ffn_tc_pair_kernel", "router_bf16_kernel"} <= kernels
    for path in PROFILES:
        name = os.path.basename(path)
        for cmd in _commands(open(path).read()):
            for args in _bench_args(cmd):
                parser.parse_args(args)          # exits (fails the test) on an unknown flag
            if cmd.startswith("ncu ") or " ncu " in cmd:
                assert "--clock-control none" in cmd, (name, cmd)
                for pat in re.findall(r"-k regex:(\S+)", cmd):
                    assert any(re.search(pat, k) for k in kernels), (name, pat)
            for script in re.findall(r"python (\S+\.py)", cmd):
                assert os.path.exists(os.path.join(ROOT, script)), (name, script)
