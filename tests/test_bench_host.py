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


def test_spectral_scaling_runs_without_plain_leading_steps():
    """The split mode's default two plain leading steps assume the Frobenius start (normalised singular values
    near 1/sqrt(m)); with spectral scaling the library rejects them, so the bench drops them by default and
    refuses an explicit request."""
    import pytest

    assert bench.plain_lead_of(bench.parse_args([])) == bench.DEFAULT_PLAIN_LEAD
    assert bench.plain_lead_of(bench.parse_args(["--spectral"])) == 0
    assert bench.plain_lead_of(bench.parse_args(["--spectral", "--plain-lead", "0"])) == 0
    with pytest.raises(SystemExit):
        bench.plain_lead_of(bench.parse_args(["--spectral", "--plain-lead", "2"]))


def test_rollup_rates_only_launches_with_known_bytes():
    """A later Lanczos A·v launch reads only the matrices still iterating, so the library states no bytes
    for it: the kernel's rate is the stated bytes over the stated launches' time, not over all of them."""
    import types

    S = types.SimpleNamespace(WORK_FLOPS=0, WORK_BYTES=1)  # the library's trace kinds
    recs = [{"name": "k_lz_matvec", "kind": 1, "work": 1e9, "nominal": 0.0, "ms": 0.2},
            {"name": "k_lz_matvec", "kind": 1, "work": 0.0, "nominal": 0.0, "ms": 0.1},
            {"name": "k_lz_matvec", "kind": 1, "work": 0.0, "nominal": 0.0, "ms": 0.1},
            {"name": "k_momentum", "kind": 1, "work": 2e9, "nominal": 0.0, "ms": 0.4}]
    _, kernels, _ = bench.rollup(S, recs, {"hbm_gbs": 6650.0}, 1590.0)
    lz = kernels["k_lz_matvec"]
    assert lz["launches"] == 3 and lz["rated_launches"] == 1
    assert abs(lz["achieved"] - 5000.0) < 1e-6  # 1 GB in 0.2 ms
    assert abs(kernels["k_momentum"]["achieved"] - 5000.0) < 1e-6 and "rated_launches" not in kernels["k_momentum"]
