"""Host-side pieces of bench.py that decide what a bench line claims: the
workload names, the algorithmic stage bytes, and the traffic entries' source
hashes. No GPU."""
import json
import os

import bench

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_workload_names_follow_the_options():
    base = bench.describe("c2_resnet50", "plain", False)
    assert base["workload"] == "resnet50_conv_set_53_layers_M4_quintic1_int8_vote"
    assert bench.describe("c2_resnet50", "plain", False, spectral=True)["workload"].endswith("_spectral_norm")
    c3 = bench.describe("c3_gpt2s", "split", True)["workload"]
    assert "local_polar" in c3 and c3.endswith("_split_bf16")


def test_stage_bytes_count_each_operand_once():
    m, n, M = 64, 256, 4
    b = bench.gemm_stage_bytes([(m, n)], M, 1, 2.0315, False, 1)
    # Gram: X (bf16) read, A (f32) and its bf16 operand written
    assert b["gram"] == M * (2 * m * n + 4 * m * m + 2 * m * m)
    # A^2: A operand read, f32 A read, B operand written
    assert b["poly"] == M * (2 * m * m + 4 * m * m + 2 * m * m)
    # B X: B and X operands read, the f32 source read, int8 signs written
    assert b["axpy"] == M * (2 * m * m + 2 * m * n + 4 * m * n + 1 * m * n)
    b2 = bench.gemm_stage_bytes([(m, n)], M, 1, 2.0315, False, 2)
    assert b2["axpy"] - b["axpy"] == M * m * n  # a bf16 U writes one byte more per entry
    bc = bench.gemm_stage_bytes([(n, m)], M, 1, 0.0, False, 1)  # tall, cubic: no A^2 stage
    assert bc["poly"] == 0 and bc["gram"] == M * (2 * m * n + 2 * m * m)


def test_committed_traffic_entries_name_existing_sources_and_profiles():
    with open(os.path.join(ROOT, "profiles", "traffic.json")) as f:
        entries = json.load(f)
    for name, e in entries.items():
        for src in e["sources"]:
            assert os.path.exists(os.path.join(ROOT, "matrix_aware_sign_b200", "csrc", src)), (name, src)
        assert os.path.exists(os.path.join(ROOT, "profiles", e["profile"])), name
        assert e["bytes_per_launch"] > 0
        # a stale hash makes the bench report null, never a number taken on other code
        got = bench.load_traffic(name)
        assert got in (None, e["bytes_per_launch"])
