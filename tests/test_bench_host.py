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
    return (f"# ncu --set full\n\nkernel sources sha256: {src_hash}\n\n"
            "## `post_rotate_fast_kernel<16, __nv_bfloat16, __nv_bfloat16>`\n\n| metric | value |\n|---|---|\n"
            "| dram__bytes_read.sum | 38.5 Mbyte |\n| dram__bytes_write.sum | 1.5 Mbyte |\n\n"
            "## `pre_rotate_fast_kernel<16, __nv_bfloat16, __nv_bfloat16>`\n\n| metric | value |\n|---|---|\n"
            "| dram__bytes_read.sum | 20.0 Mbyte |\n| dram__bytes_write.sum | 2.0 Mbyte |\n")


@pytest.fixture
def fake_root(tmp_path, monkeypatch):
    """A repository root with the real CUDA sources and a profiles/ folder."""
    real = os.path.join(bench.ROOT, "ternary_butterfly_experts_b200", "csrc")
    shutil.copytree(real, tmp_path / "ternary_butterfly_experts_b200" / "csrc")
    (tmp_path / "profiles").mkdir()
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    return tmp_path


def test_traffic_read_only_for_the_current_sources(fake_root):
    path = fake_root / "profiles" / "ncu_full_rotations_d512_n256.md"
    path.write_text(_summary(bench.kernel_sources_hash()))
    assert bench.profiled_traffic("post_rotate", "d512_n256") == pytest.approx(40.0e6)
    assert bench.profiled_traffic("pre_rotate", "d512_n256") == pytest.approx(22.0e6)
    assert bench.profiled_traffic("combine", "d512_n256") is None          # not in the summary
    assert bench.profiled_traffic("post_rotate", "d1024_n256") is None     # another workload
    path.write_text(_summary("0" * 64))                                     # taken from other sources
    assert bench.profiled_traffic("post_rotate", "d512_n256") is None


def test_source_hash_follows_the_sources(fake_root):
    before = bench.kernel_sources_hash()
    with open(fake_root / "ternary_butterfly_experts_b200" / "csrc" / "combine_probe.cuh", "w") as f:
        f.write("// a new source file\n")
    assert bench.kernel_sources_hash() != before
