"""The benchmark's arithmetic on CPU: the algorithmic bytes and FLOPs that the
roofline divides by, checked against the shape arithmetic of the Mixtral layer
(three 4,096 x 14,336 matrices per expert; active FLOPs 6 T K d ffn), and the
traffic records that bench.py reads back from profiles/."""
import os

import numpy as np
import pytest

import bench
import moe_inputs as mi


def all_touched(cfg):
    return np.full(cfg.n, 1, np.int64)


def test_decode_bytes_are_the_touched_weights():
    cfg = mi.CONFIGS["decode"]
    w = bench.algorithmic(cfg, all_touched(cfg))
    per_expert = 3 * 4096 * 14336                       # parameters of one expert
    assert per_expert == 176_160_768
    weights = 8 * per_expert * 2                         # bf16
    assert w["layer_bytes"] == weights + 32 * 4096 * 2 * 2 + 4096 * 8 * 4
    assert abs(weights / 1e9 - 2.8186) < 1e-4
    # GEMM1 moves w1 and w3 (two thirds of the weights) plus its activations
    assert w["gemm1"]["bytes"] == 2 * weights // 3 + 64 * 4096 * 2 + 64 * 14336 * 2
    assert w["gemm2"]["bytes"] == weights // 3 + 64 * 14336 * 2 + 64 * 4096 * 2


def test_active_flops_follow_the_shapes():
    cfg = mi.CONFIGS["prefill"]
    w = bench.algorithmic(cfg, all_touched(cfg))
    R = 4096 * 2
    assert w["gemm1"]["flops"] == 4.0 * R * 4096 * 14336
    assert w["gemm2"]["flops"] == 2.0 * R * 14336 * 4096
    assert w["active_flops"] == w["gemm1"]["flops"] + w["gemm2"]["flops"] + 2.0 * 4096 * 4096 * 8
    assert abs(w["active_flops"] / 1e12 - 2.886) < 1e-3


def test_untouched_experts_move_no_weight_bytes():
    cfg = mi.CONFIGS["decode"]
    counts = np.zeros(cfg.n, np.int64)
    counts[[1, 5]] = 7
    two = bench.algorithmic(cfg, counts)
    eight = bench.algorithmic(cfg, all_touched(cfg))
    assert two["experts_touched"] == 2
    per_expert = 3 * 4096 * 14336 * 2
    assert eight["layer_bytes"] - two["layer_bytes"] == 6 * per_expert


@pytest.mark.parametrize("experts,bytes_per_weight", [("e4m3", 1.0), ("fp4", 0.5625), ("w4a4", 0.5625)])
def test_low_precision_weight_bytes(experts, bytes_per_weight):
    cfg = mi.CONFIGS["decode"]
    w = bench.algorithmic(cfg, all_touched(cfg), experts)
    weights = 8 * 3 * 4096 * 14336
    wbytes = w["layer_bytes"] - 32 * 4096 * 2 * 2 - 4096 * 8 * 4
    # codes (and block scales) per weight, plus the per-column or per-matrix scales
    assert abs(wbytes / weights - bytes_per_weight) < 2e-3


def test_traffic_record_is_used_only_for_the_profiled_source(tmp_path, monkeypatch):
    src = tmp_path / "sparse_mixture_experts_24_b200" / "csrc"
    src.mkdir(parents=True)
    (src / "gemm_tc.cu").write_text("kernel source A")
    (src / "gemm_w4a4.cu").write_text("kernel source B")
    (src / "gemm_tc3.cu").write_text("kernel source C")
    sha_a = bench.source_sha(str(src / "gemm_tc.cu"))
    sha_b = bench.source_sha(str(src / "gemm_w4a4.cu"))
    sha_c = bench.source_sha(str(src / "gemm_tc3.cu"))
    prof = tmp_path / "profiles"
    prof.mkdir()
    (prof / "ncu_traffic.txt").write_text(
        "# comment\n"
        "traffic gemm1 decode 123 src_sha=%s\n"
        "traffic gemm1 decode_w4a4 456 src_sha=%s\n"
        "traffic gemm1 prefill 789 src_sha=0000000000000000\n"
        "traffic gemm2 prefill 321 src_sha=%s file=gemm_tc3.cu\n" % (sha_a, sha_b, sha_c))
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    assert bench.recorded_traffic("gemm1", "decode") == 123.0
    assert bench.recorded_traffic("gemm1", "decode_w4a4") == 456.0
    assert bench.recorded_traffic("gemm1", "prefill") is None          # taken on another source
    assert bench.recorded_traffic("gemm2", "decode") is None           # never recorded
    assert bench.recorded_traffic("gemm2", "prefill") == 321.0         # the line's own source file
    (src / "gemm_tc.cu").write_text("kernel source A, changed")
    assert bench.recorded_traffic("gemm1", "decode") is None           # stale after a change
    assert bench.recorded_traffic("gemm2", "prefill") == 321.0
    (src / "gemm_tc3.cu").write_text("kernel source C, changed")
    assert bench.recorded_traffic("gemm2", "prefill") is None


def test_committed_traffic_records_parse():
    path = os.path.join(bench.ROOT, "profiles", "ncu_traffic.txt")
    lines = [l.split() for l in open(path) if l.startswith("traffic ")]
    assert lines, "no traffic records"
    for parts in lines:
        assert len(parts) in (5, 6) and parts[4].startswith("src_sha=") and float(parts[3]) > 0
        assert len(parts) == 5 or parts[5].startswith("file=")


def test_committed_traffic_records_name_the_current_sources():
    """Every committed traffic record was taken on the kernel source as it is
    now: a kernel edited since its ncu capture would report no traffic."""
    path = os.path.join(bench.ROOT, "profiles", "ncu_traffic.txt")
    stale = []
    for line in open(path):
        if line.startswith("traffic "):
            parts = line.split()
            if bench.recorded_traffic(parts[1], parts[2]) != float(parts[3]):
                stale.append(line.strip())
    assert not stale, stale
