"""The ncu summariser (raw CSV -> the JSON bench.py reads), on synthetic
ncu output (no GPU, no ncu)."""
import json

from ternary_butterfly_experts_b200 import ncu_summary as S

RAW = (
    '"ID","Kernel Name","gpu__time_duration.sum","dram__bytes_read.sum","dram__bytes_write.sum",'
    '"launch__registers_per_thread","smsp__average_warps_issue_stalled_long_scoreboard_per_issue_active.ratio",'
    '"smsp__average_warps_issue_stalled_wait_per_issue_active.ratio","other"\n'
    '"","","us","Mbyte","Kbyte","register/thread","",""," "\n'
    '"0","void bfmoe::fused_expert_kernel<512>(CUtensorMap_st, const __nv_bfloat16 *)","94.2","26.8","1059.84",'
    '"96","4.5","1.4","x"\n'
    '"1","void bfmoe::fused_expert_kernel<512>(CUtensorMap_st, const __nv_bfloat16 *)","99.0","30.0","1.0",'
    '"96","4.0","1.0","x"\n'
)

LAUNCHES = (
    '"ID","Kernel Name","Metric Name","Metric Unit","Metric Value"\n'
    '"0","void bfmoe::router_tc_kernel<128, 3, 2>(CUtensorMap_st)","gpu__time_duration.sum","ns","24000"\n'
    '"1","void bfmoe::fused_expert_kernel<512>(CUtensorMap_st)","gpu__time_duration.sum","ns","90000"\n'
    '"2","void bfmoe::router_tc_kernel<128, 3, 2>(CUtensorMap_st)","gpu__time_duration.sum","ns","26000"\n'
    '"3","void bfmoe::fused_expert_kernel<512>(CUtensorMap_st)","gpu__time_duration.sum","usecond","91"\n'
)


def test_full_summary_keeps_first_launch_and_dram_bytes(tmp_path):
    raw = tmp_path / "raw.csv"
    raw.write_text(RAW)
    js = S.summarize_full(str(raw), "d512_n256", "ncu --set full ...")
    assert list(js["kernels"]) == ["fused_expert_kernel<512>"]
    e = js["kernels"]["fused_expert_kernel<512>"]
    assert e["dram_bytes_per_launch"] == 26.8e6 + 1059.84e3   # first launch only, units applied
    assert e["duration_us"] == 94.2
    assert e["metrics"]["launch__registers_per_thread"]["value"] == 96
    assert list(e["top_stalls_per_issue"]) == ["long_scoreboard", "wait"]
    assert js["kernel_sources_sha256"] == S.kernel_sources_hash()
    md = S.to_markdown(js)
    assert "fused_expert_kernel<512>" in md and "ncu --set full ..." in md


def test_launch_list_totals_and_shares(tmp_path):
    p = tmp_path / "l.csv"
    p.write_text(LAUNCHES)
    js = S.summarize_launches(str(p), "d512_n256", "ncu --metrics gpu__time_duration.sum ...")
    k = js["kernels"]
    assert k["fused_expert_kernel<512>"]["launches"] == 2
    assert k["fused_expert_kernel<512>"]["total_us"] == 181.0
    assert k["router_tc_kernel<128, 3, 2>"]["avg_us"] == 25.0
    assert abs(sum(e["share"] for e in k.values()) - 1.0) < 1e-12
    assert list(k)[0] == "fused_expert_kernel<512>"          # sorted by total time
    json.dumps(js)


def test_cli_writes_json_and_markdown(tmp_path):
    raw = tmp_path / "raw.csv"
    raw.write_text(RAW)
    out = tmp_path / "ncu_fused_expert_d512_n256"
    assert S.main(["full", "--raw", str(raw), "--workload", "d512_n256", "--command", "c", "--out", str(out)]) == 0
    assert json.loads((tmp_path / "ncu_fused_expert_d512_n256.json").read_text())["workload"] == "d512_n256"
    assert (tmp_path / "ncu_fused_expert_d512_n256.md").read_text().startswith("# ncu --set full")
