"""Host-side arithmetic of bench.py (no GPU): the algorithmic bytes and
operations behind every roofline fraction, the bound decision, the target
summary and the digest check that guards the profiled DRAM traffic."""
import json

import pytest

import bench


def test_weight_bytes_of_the_4096_square_layer():
    # 4-bit codes + one (s_u8, a) byte pair per 64-weight group + an fp32
    # channel scale: 8 388 608 + 524 288 + 16 384 bytes
    assert bench.weight_bytes(4096, 4096) == 8929280
    assert bench.gemm_bytes(1, 4096, 4096) == 8929280 + 4096 + 4 + 2 * 4096
    assert bench.gemm_ops(3, 5, 7) == 2 * 3 * 5 * 7
    assert bench.act_bytes(2, 4096) == 5 * 2 * 4096 + 8


def test_bound_switches_from_hbm_to_tensor_at_the_ridge():
    peaks = {"hbm": 6546.9, "int8": 3210.0}
    # ridge = 3210e12 / 6546.9e9 ~ 490 ops per byte; on 4096 x 4096, M = 128
    # does 409 ops per algorithmic byte (HBM-bound) and M = 256 711 (tensor)
    b128, f128 = bench.bound_and_frac(128, 4096, 4096, 10e-6, peaks)
    assert b128 == "hbm"
    assert abs(f128 - bench.gemm_bytes(128, 4096, 4096) / (6546.9e9 * 10e-6)) < 1e-12
    assert bench.bound_and_frac(256, 4096, 4096, 10e-6, peaks)[0] == "tensor"
    b8k, f8k = bench.bound_and_frac(8192, 8192, 8192, 400e-6, peaks)
    assert b8k == "tensor"
    assert abs(f8k - bench.gemm_ops(8192, 8192, 8192) / (3210.0e12 * 400e-6)) < 1e-12


def test_target_summary_leaves_out_the_tiny_case_and_takes_extremes():
    cases = [
        {"workload": "tiny", "M": 16, "bound": "hbm", "frac": 0.004},
        {"workload": "w", "M": 1, "bound": "hbm", "frac": 0.5},
        {"workload": "w", "M": 16, "bound": "hbm", "frac": 0.7},
        {"workload": "w", "M": 32, "bound": "hbm", "frac": 0.1},      # M > 16: not counted
        {"workload": "p", "M": 8192, "bound": "tensor", "frac": 0.85},
        {"workload": "p", "M": 16384, "bound": "tensor", "frac": 0.8},
        {"workload": "p", "M": 2048, "bound": "tensor", "frac": 0.9},  # M < 4096: not counted
    ]
    t = bench.target_summary(cases)
    assert t["hbm_frac_at_M_le_16"]["min"] == 0.5
    assert t["hbm_frac_at_M_le_16"]["max"] == 0.7
    assert t["hbm_frac_at_M_le_16"]["cases"] == 2
    assert "tiny" in t["hbm_frac_at_M_le_16"]["excluded"]
    assert t["int8_frac_at_M_ge_4096"]["min"] == 0.8
    assert t["int8_frac_at_M_ge_4096"]["max"] == 0.85


def test_profiled_traffic_only_for_the_sources_it_was_taken_on(tmp_path, monkeypatch):
    prof = tmp_path / "profiles"
    prof.mkdir()
    (prof / "gemm_traffic.json").write_text(json.dumps(
        {"csrc_digest": "0123456789abcdef", "sweep_mean_dram_bytes_per_launch": 1.0}))
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    monkeypatch.setattr(bench, "csrc_digest", lambda: "0123456789abcdef")
    assert bench.profiled_traffic()["sweep_mean_dram_bytes_per_launch"] == 1.0
    monkeypatch.setattr(bench, "csrc_digest", lambda: "fedcba9876543210")
    assert bench.profiled_traffic() is None


def test_committed_traffic_summary_is_consistent():
    # the committed ncu summary, when it was taken on the kernels in the tree
    # (else the bench line reports no traffic and there is nothing to check)
    d = bench.profiled_traffic()
    if d is None:
        pytest.skip("profiles/gemm_traffic.json was taken on other kernel sources")
    per = d["per_m"]
    assert [x["M"] for x in per] == [1, 2, 4, 8, 16, 32, 64, 128, 256]
    for x in per:
        assert x["algorithmic"] == bench.gemm_bytes(x["M"], 4096, 4096)
        # every launch reads its weights once: DRAM bytes within 20% of the
        # algorithmic bytes (the bf16 output stays in L2)
        assert 0.8 < (x["dram_read"] + x["dram_write"]) / x["algorithmic"] < 1.05
