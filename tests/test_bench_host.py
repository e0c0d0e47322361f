"""Host-side pieces of bench.py: the algorithmic bytes it divides by, the DRAM-traffic record it
reports, and the config both arms print. No GPU."""

import json
import os

import bench


def test_stack_bytes_match_the_shapes():
    shapes = bench.stack_shapes()
    assert len(shapes) == 256
    # 64 x {QKV 7168x5120, O 5120x5120, gate+up 34816x5120, down 5120x17408}: codes N*K/2 and
    # scales N*K/16 bytes per matrix
    weights = 64 * (7168 * 5120 + 5120 * 5120 + 34816 * 5120 + 5120 * 17408)
    assert sum(N * K for (_, _, _, N, K, _) in shapes) == weights == 21_139_292_160
    assert weights // 2 + weights // 16 == 11_890_851_840          # codes + block scales
    assert bench.w_bytes(shapes) == 11_890_851_840 + 4 * 256        # + one fp32 tensor scale each
    # per pass: X in (2 M K) and Y out (2 M N) for every matrix
    for M in (1, 17, 32):
        xy = sum(2 * M * K + 2 * M * N for (_, _, _, N, K, _) in shapes)
        assert xy == M * 10_878_976
        assert bench.pass_bytes(shapes, M) == bench.w_bytes(shapes) + xy


def test_traffic_record_matches_the_sources_and_scales_per_M():
    shapes = bench.stack_shapes()
    rec = json.load(open(os.path.join(bench.ROOT, "profiles", "traffic.json")))
    assert rec["source_hash"] == bench.source_hash("exact"), "traffic.json was taken on other sources"
    t = bench.profiled_traffic(shapes, "exact")
    mean_alg = sum(bench.pass_bytes(shapes, M) for M in bench.M_SWEEP) / len(bench.M_SWEEP)
    ratios = [v["ratio"] for v in rec["per_M"].values()]
    assert min(ratios) * mean_alg * 0.999 <= t <= max(ratios) * mean_alg * 1.001
    # a record for another path's kernels is not used
    assert bench.profiled_traffic(shapes, "block-scaled") is None


def test_both_arms_print_the_same_config():
    a = bench.arm_config("exact", 1)
    b = bench.arm_config("exact", 1)
    assert a == b and a["w_bytes"] == 11_890_851_840 + 4 * 256 and a["matrices"] == 256
    assert bench.arm_config("exact", 8)["parallelism"] == "replicas x8"


def test_head_and_gdn_bytes():
    assert bench.head_bytes(1) == 151936 * 5120 + 4 * 151936 + 2 * 5120 + 4 * 151936 + 16
    assert bench.GDN_H == 1536 and bench.GDN_D == 128
    assert round(bench.FP32_FMA_PEAK_TFLOPS, 1) == 74.4
