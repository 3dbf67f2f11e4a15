"""Host-side arithmetic of bench.py: algorithmic work per kernel, the peak a
roofline entry is measured against, and the source-hash gate on the DRAM
traffic read from the ncu summaries (no GPU)."""
import os
import shutil

import pytest

import bench
import workloads as W


def _tables_bytes(wl):
    return wl.n_experts * wl.stages * (wl.d // 2) * 8


def test_post_rotation_bytes_on_the_headline():
    wl = W.WORKLOADS["d512_n256"]
    costs = bench.kernel_costs(wl, _tables_bytes(wl))
    bound, work, unit = costs["post_rotate"]
    # Z read and gated slots written, bf16, 32768 rows of 512; plus the phi table
    assert (bound, unit) == ("hbm", "GB/s")
    assert work == 2 * 32768 * 512 * 2 + 256 * 9 * 256 * 8 == 71_827_456


def test_gemm_flops_and_path_roofline_bytes():
    wl = W.WORKLOADS["d1024_n256"]
    bound, work, _ = bench.kernel_costs(wl, _tables_bytes(wl))["ternary_gemm_tc"]
    assert bound == "tensor" and work == 2.0 * 65536 * 2 * 1024 * 1024
    # x in and y out once, 2-bit base, both angle sets, gate weights and bias, routing
    expect = 2 * 65536 * 1024 * 2 + 1024 * 1024 // 4 + 2 * 256 * 10 * 512 * 4 + 256 * 1024 * 4 + 256 * 4 + 65536 * 2 * 8
    assert bench.algorithmic_bytes(wl) == expect


PEAKS = {"hbm_gbs": 6000.0, "bf16_tflops": 1600.0, "bf16_tflops_sustained": 1400.0}


def test_roofline_peak_choice():
    wl = W.WORKLOADS["d512_n256"]
    costs = bench.kernel_costs(wl, _tables_bytes(wl))
    one_ms = (1, 1.0)  # one launch of 1 ms
    burst = bench.roofline_entry("ternary_gemm_tc", one_ms, costs, PEAKS, {})
    sustained = bench.roofline_entry("ternary_gemm_tc", one_ms, costs, PEAKS, {}, sustained=True)
    assert burst["peak"] == 1600.0 and sustained["peak"] == 1400.0
    assert burst["achieved"] == pytest.approx(costs["ternary_gemm_tc"][1] / 1e-3 / 1e12)
    assert sustained["frac"] == pytest.approx(sustained["achieved"] / 1400.0)
    hbm = bench.roofline_entry("post_rotate", (2, 0.07), costs, PEAKS, {}, sustained=True)
    # an HBM-bound kernel keeps the copy bandwidth; 2 launches in 0.07 ms
    assert hbm["peak"] == 6000.0 and hbm["avg_launch_us"] == pytest.approx(35.0)
    assert hbm["achieved"] == pytest.approx(71_827_456 / 35e-6 / 1e9)


def _summary(src_hash):
    return {"kind": "ncu --set full", "workload": "d512_n256", "command": "ncu ...",
            "kernel_sources_sha256": src_hash,
            "kernels": {"fused_expert_kernel<512>": {"dram_bytes_per_launch": 27.9e6},
                        "router_tc_kernel<128, 3, 2>": {"dram_bytes_per_launch": 17.6e6}}}


@pytest.fixture
def fake_root(tmp_path, monkeypatch):
    """A repository root with the real CUDA sources and a profiles/ folder."""
    real = os.path.join(bench.ROOT, "ternary_butterfly_experts_b200", "csrc")
    shutil.copytree(real, tmp_path / "ternary_butterfly_experts_b200" / "csrc")
    (tmp_path / "profiles").mkdir()
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    return tmp_path


def test_traffic_read_only_for_the_current_sources(fake_root):
    import json
    path = fake_root / "profiles" / "ncu_fused_expert_d512_n256.json"
    path.write_text(json.dumps(_summary(bench.kernel_sources_hash())))
    assert bench.profiled_traffic("fused_expert", "d512_n256") == pytest.approx(27.9e6)
    assert bench.profiled_traffic("router_tc", "d512_n256") == pytest.approx(17.6e6)
    assert bench.profiled_traffic("combine", "d512_n256") is None          # not in the summary
    assert bench.profiled_traffic("fused_expert", "d1024_n256") is None    # another workload
    path.write_text(json.dumps(_summary("0" * 64)))                         # taken from other sources
    assert bench.profiled_traffic("fused_expert", "d512_n256") is None


def test_source_hash_follows_the_sources(fake_root):
    before = bench.kernel_sources_hash()
    with open(fake_root / "ternary_butterfly_experts_b200" / "csrc" / "combine_probe.cuh", "w") as f:
        f.write("// a new source file\n")
    assert bench.kernel_sources_hash() != before


def test_as_built_traffic_is_listed_apart():
    wl = W.WORKLOADS["d512_n256"]
    ab = bench.as_built_bytes(wl)
    # the fused path keeps X_rot and Z on chip; the slot buffer and the logits remain
    assert "x_rot_round_trip" not in ab and "z_round_trip" not in ab
    assert ab["slot_buffer"] == 2 * 32768 * 512 * 2
    assert ab["router_logits_f32"] == 16384 * 256 * 4
    assert ab["total"] == sum(v for k, v in ab.items() if k != "total")
    ab4 = bench.as_built_bytes(W.WORKLOADS["d2048_n1024"])
    assert ab4["x_rot_round_trip"] == 2 * 131072 * 4 * 2048 * 2
