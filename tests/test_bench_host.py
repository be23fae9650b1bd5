"""The benchmark's host-side accounting (no GPU): the algorithmic bytes and
FLOPs it divides by, its launch counts, the imbalance score, and the rule by
which an ncu traffic record stays valid only for the code it was taken on."""
import json

import bench
import synth


def test_algorithmic_bytes_and_flops_of_the_workloads():
    dec, pre = synth.CONFIGS["decode"], synth.CONFIGS["prefill"]
    # the used experts' three matrices once (64 routed + 4 shared, bf16), the
    # router, x in and y out
    want = 2 * (68 * 3 * 1344 * 5120 + 64 * 5120 + 2 * 456 * 5120)
    assert bench.layer_bytes(dec, 64) == want == 2817556480
    # 8-bit: one byte per weight plus an fp32 scale per weight row
    want8 = 68 * (3 * 1344 * 5120 + 4 * (2 * 1344 + 5120)) + 2 * (64 * 5120 + 2 * 456 * 5120)
    assert bench.layer_bytes_fp8(dec, 64) == want8 == 1415899136
    # 2 * rows * d * 3I over the routed and shared rows
    assert bench.ffn_flops(pre) == 2.0 * (4096 * 8 + 4 * 4096) * 5120 * 3 * 1344
    assert abs(bench.ffn_flops(pre) / 1e12 - 2.0295) < 1e-3
    assert bench.layer_flops(pre) == bench.ffn_flops(pre) + 2.0 * 4096 * 5120 * 64
    # a training step: the forward, twice the FFN's expert GEMMs, three router GEMMs
    assert bench.train_flops(pre) == (bench.layer_flops(pre) + 2 * bench.ffn_flops(pre)
                                      + 6 * 4096 * 64 * 5120)
    # fewer used experts, fewer bytes
    assert bench.layer_bytes(dec, 60) == want - 2 * 4 * 3 * 1344 * 5120


def test_launch_counts_follow_the_library_rules():
    dec, pre = synth.CONFIGS["decode"], synth.CONFIGS["prefill"]
    assert bench.layer_launches(dec) == 4              # permute inside the FFN launch
    assert bench.layer_launches(dec, fp8=True) == 5    # 8-bit paths: a launch of their own
    assert bench.layer_launches(pre) == 5              # above 8192 routed rows
    assert bench.layer_launches(synth.CONFIGS["tiny"]) == 5   # fp32


def test_imbalance_score():
    eq = bench.imbalance_score([3, 1, 2, 2] * 2, 2, 16)
    assert eq == {"score": 0.0, "group_loads": [8, 8]}
    skew = bench.imbalance_score([4, 4, 0, 0], 2, 8)
    assert skew["score"] == 1.0 and skew["group_loads"] == [8, 0]


def test_code_hash_ignores_comments_only():
    src = 'int a = 1; // note\n/* block\n comment */ const char *s = "x//y"; char c = \'/\';\n'
    edited = src.replace("note", "another note").replace("block", "other")
    assert bench.code_of(src) == bench.code_of(edited)
    assert '"x//y"' in bench.code_of(src)
    assert bench.code_of(src) != bench.code_of(src.replace("a = 1", "a = 2"))


def _record_file(tmp_path, rec):
    p = tmp_path / "record.md"
    p.write_text("# a capture\n\ntraffic-record: %s\n" % json.dumps(rec))
    return str(p)


def test_traffic_record_is_valid_only_on_its_sources(tmp_path, monkeypatch):
    files = ["common.cuh"]
    good = {"kernel": "k", "workload": "w", "dram_bytes_per_launch": 123, "files": files,
            "src_sha16": bench.source_sha16(files)}
    monkeypatch.setattr(bench, "TRAFFIC_RECORDS", (_record_file(tmp_path, good),))
    n, why = bench.traffic_record("k", "w")
    assert n == 123 and "ncu" in why
    assert bench.traffic_record("k", "other")[0] is None
    assert bench.traffic_record("other", "w")[0] is None

    stale = dict(good, src_sha16="0" * 16)
    monkeypatch.setattr(bench, "TRAFFIC_RECORDS", (_record_file(tmp_path, stale),))
    n, why = bench.traffic_record("k", "w")
    assert n is None and "kernel changed" in why
