"""Condense ncu output into the small JSON (and markdown) summaries kept under
profiles/, which bench.py reads back for its DRAM-traffic figure.

    python -m ternary_butterfly_experts_b200.ncu_summary full \\
        --raw prof.csv --workload d512_n256 --command "<the ncu command>" \\
        --out profiles/ncu_fused_expert_d512_n256
    python -m ternary_butterfly_experts_b200.ncu_summary launches \\
        --csv launches.csv --workload d512_n256 --command "<the ncu command>" \\
        --out profiles/launches_d512_n256

``full`` reads ``ncu -i <report> --page raw --csv`` (a header row, a units
row, one row per captured launch) and keeps the first launch of each kernel;
``launches`` reads the ``--csv --log-file`` output of a
``--metrics gpu__time_duration.sum`` run (one row per launch and metric).
Each writes <out>.json and <out>.md.  The JSON records the sha256 of the
library's CUDA sources at the time of writing: bench.py only uses a summary
whose hash matches the sources it runs.
"""
from __future__ import annotations

import argparse
import csv
import hashlib
import json
import os
import re

CSRC = os.path.join(os.path.dirname(os.path.abspath(__file__)), "csrc")

# Metrics kept from a --set full capture (those present in the capture).
FULL_METRICS = [
    "gpu__time_duration.sum",
    "dram__bytes_read.sum",
    "dram__bytes_write.sum",
    "gpu__dram_throughput.avg.pct_of_peak_sustained_elapsed",
    "lts__t_sectors_srcunit_tex_op_read.sum",
    "lts__throughput.avg.pct_of_peak_sustained_elapsed",
    "sm__pipe_tensor_cycles_active.avg.pct_of_peak_sustained_elapsed",
    "sm__pipe_fma_cycles_active.avg.pct_of_peak_sustained_active",
    "sm__pipe_alu_cycles_active.avg.pct_of_peak_sustained_active",
    "sm__inst_executed_pipe_lsu.avg.pct_of_peak_sustained_active",
    "sm__throughput.avg.pct_of_peak_sustained_elapsed",
    "sm__warps_active.avg.pct_of_peak_sustained_active",
    "smsp__issue_active.avg.pct_of_peak_sustained_active",
    "sm__inst_executed.avg.per_cycle_active",
    "launch__registers_per_thread",
    "launch__grid_size",
    "launch__block_size",
]
STALL_PREFIX = "smsp__average_warps_issue_stalled_"
STALL_SUFFIX = "_per_issue_active.ratio"

# Bytes per unit ncu may print.
_SCALE = {"byte": 1, "Kbyte": 1e3, "Mbyte": 1e6, "Gbyte": 1e9, "KB": 1e3, "MB": 1e6, "GB": 1e9,
          "ns": 1e-3, "us": 1.0, "usecond": 1.0, "msecond": 1e3, "ms": 1e3, "nsecond": 1e-3}


def kernel_sources_hash(csrc: str = CSRC) -> str:
    """sha256 over the library's CUDA sources (the .cu / .cuh files of
    `csrc`), sorted by name."""
    h = hashlib.sha256()
    for f in sorted(os.listdir(csrc)):
        if f.endswith((".cu", ".cuh")):
            h.update(f.encode())
            with open(os.path.join(csrc, f), "rb") as fh:
                h.update(fh.read())
    return h.hexdigest()


def short_name(kernel: str) -> str:
    """`void ns::foo_kernel<512>(...)` -> `foo_kernel<512>`."""
    k = re.sub(r"^void\s+", "", kernel.strip())
    k = k.split("(")[0]
    return k.split("::")[-1]


def _num(v: str):
    try:
        return float(v.replace(",", ""))
    except ValueError:
        return None


def parse_full(raw_csv: str):
    """{kernel: {metric: (value, unit)}} for the first launch of each kernel."""
    with open(raw_csv, newline="") as f:
        rows = [r for r in csv.reader(f) if r]
    # the header row names "Kernel Name"; the next row holds the units
    hi = next(i for i, r in enumerate(rows) if "Kernel Name" in r)
    hdr, units = rows[hi], rows[hi + 1]
    out = {}
    for r in rows[hi + 2:]:
        if len(r) != len(hdr):
            continue
        d = dict(zip(hdr, r))
        name = short_name(d["Kernel Name"])
        if name in out:
            continue
        m = {}
        for col, unit, val in zip(hdr, units, r):
            if col in FULL_METRICS or (col.startswith(STALL_PREFIX) and col.endswith(STALL_SUFFIX)):
                x = _num(val)
                if x is not None:
                    m[col] = (x, unit)
        out[name] = m
    return out


def summarize_full(raw_csv: str, workload: str, command: str):
    kern = parse_full(raw_csv)
    js = {"kind": "ncu --set full", "workload": workload, "command": command,
          "kernel_sources_sha256": kernel_sources_hash(), "kernels": {}}
    for name, m in kern.items():
        e = {"metrics": {k: {"value": v, "unit": u} for k, (v, u) in m.items() if not k.startswith(STALL_PREFIX)}}
        stalls = sorted(((k[len(STALL_PREFIX):-len(STALL_SUFFIX)], v) for k, (v, _) in m.items()
                         if k.startswith(STALL_PREFIX)), key=lambda kv: -kv[1])
        e["top_stalls_per_issue"] = dict(stalls[:6])
        rd, wr = m.get("dram__bytes_read.sum"), m.get("dram__bytes_write.sum")
        if rd and wr:
            e["dram_bytes_per_launch"] = rd[0] * _SCALE.get(rd[1], 1) + wr[0] * _SCALE.get(wr[1], 1)
        t = m.get("gpu__time_duration.sum")
        if t:
            e["duration_us"] = t[0] * _SCALE.get(t[1], 1)
        js["kernels"][name] = e
    return js


def summarize_launches(launch_csv: str, workload: str, command: str):
    with open(launch_csv, newline="") as f:
        rows = [r for r in csv.reader(f) if r]
    hi = next(i for i, r in enumerate(rows) if "Kernel Name" in r)
    hdr = rows[hi]
    per = {}
    order = []
    for r in rows[hi + 1:]:
        if len(r) != len(hdr):
            continue
        d = dict(zip(hdr, r))
        if d.get("Metric Name") != "gpu__time_duration.sum":
            continue
        v = _num(d.get("Metric Value", ""))
        if v is None:
            continue
        us = v * _SCALE.get(d.get("Metric Unit", "ns"), 1e-3)
        name = short_name(d["Kernel Name"])
        if name not in per:
            per[name] = [0, 0.0]
            order.append(name)
        per[name][0] += 1
        per[name][1] += us
    total = sum(t for _, t in per.values()) or 1.0
    js = {"kind": "ncu launch list (gpu__time_duration.sum; cold-cache, serialised: compare shares)",
          "workload": workload, "command": command, "kernel_sources_sha256": kernel_sources_hash(),
          "kernels": {n: {"launches": per[n][0], "total_us": per[n][1], "avg_us": per[n][1] / per[n][0],
                          "share": per[n][1] / total} for n in sorted(order, key=lambda n: -per[n][1])}}
    return js


def to_markdown(js) -> str:
    lines = [f"# {js['kind']} — {js['workload']}", "",
             f"kernel sources sha256: {js['kernel_sources_sha256']}", "", "Command:", "", "```",
             js["command"], "```", ""]
    if "launch list" in js["kind"]:
        lines += ["| kernel | launches | total µs | avg µs | share |", "|---|---|---|---|---|"]
        for n, e in js["kernels"].items():
            lines.append(f"| `{n}` | {e['launches']} | {e['total_us']:.1f} | {e['avg_us']:.2f} | {e['share']:.3f} |")
    else:
        for n, e in js["kernels"].items():
            lines += [f"## `{n}`", "", "| metric | value |", "|---|---|"]
            for k, mv in e["metrics"].items():
                lines.append(f"| {k} | {mv['value']:g} {mv['unit']} |")
            if "dram_bytes_per_launch" in e:
                lines.append(f"| DRAM bytes per launch (read + write) | {e['dram_bytes_per_launch']:.4g} |")
            lines += ["", "Top stalls (warps per issue): " +
                      ", ".join(f"{k} {v:.2f}" for k, v in e["top_stalls_per_issue"].items()), ""]
    return "\n".join(lines) + "\n"


def main(argv=None):
    ap = argparse.ArgumentParser(description=__doc__.split("\n")[0])
    sub = ap.add_subparsers(dest="mode", required=True)
    f = sub.add_parser("full")
    f.add_argument("--raw", required=True)
    l_ = sub.add_parser("launches")
    l_.add_argument("--csv", required=True)
    for p in (f, l_):
        p.add_argument("--workload", required=True)
        p.add_argument("--command", required=True)
        p.add_argument("--out", required=True, help="output path without extension")
    a = ap.parse_args(argv)
    js = summarize_full(a.raw, a.workload, a.command) if a.mode == "full" else \
        summarize_launches(a.csv, a.workload, a.command)
    with open(a.out + ".json", "w") as fh:
        json.dump(js, fh, indent=1)
    with open(a.out + ".md", "w") as fh:
        fh.write(to_markdown(js))
    return 0


if __name__ == "__main__":
    raise SystemExit(main())
