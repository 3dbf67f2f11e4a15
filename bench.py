"""Throughput of the ButterflyMoE expert forward (router + forward) on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl ours|reference]

One JSON line on rank 0.  A step is one router + forward pass over one batch
of the named synthetic workload (default: d=512, N=256 experts, top-2,
T=16384 bf16 tokens).  Inputs are resident in HBM before the timed region;
L2 is flushed (a 512 MiB write) between timed steps, outside the timed
intervals.  Each step is timed with CUDA events on the launching stream; the
total is the max over ranks.  With N > 1 GPUs every rank runs its own batch
(tokens shard with no collective on the data path; weights are replicated):
"scaling": "weak".

``--impl reference`` times the CPU float64 oracle (test infrastructure) on the
host cores instead, on bounded samples of the same workload.
"""
from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import subprocess
import sys
import tempfile
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import workloads as W  # noqa: E402

METRIC = "routed tokens/sec (bf16, d=512, N=256, top-2)"
UNIT = "tokens/s"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0,
                  "sm_max_mhz": 1965.0}
SM_COUNT = 148
FP32_LANES_PER_SM = 128


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


def physical_gpu_index(local: int) -> int:
    vis = os.environ.get("CUDA_VISIBLE_DEVICES", "")
    ids = [v for v in vis.split(",") if v.strip()]
    if ids and local < len(ids) and ids[local].strip().isdigit():
        return int(ids[local])
    return local


def dist_env():
    return int(os.environ.get("RANK", "0")), int(os.environ.get("WORLD_SIZE", "1")), \
        int(os.environ.get("LOCAL_RANK", "0"))


# ---------------------------------------------------------------------------
# Clock sampling during the timed region
# ---------------------------------------------------------------------------
class ClockSampler:
    QUERY = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu_index = gpu_index
        self.proc = None
        self.path = None

    def __enter__(self):
        try:
            fd, self.path = tempfile.mkstemp(suffix=".csv")
            os.close(fd)
            self.fh = open(self.path, "w")
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.QUERY}", "--format=csv,noheader,nounits", "-lms", "100",
                 "-i", str(self.gpu_index)], stdout=self.fh, stderr=subprocess.DEVNULL)
            time.sleep(0.3)
        except (OSError, FileNotFoundError):
            self.proc = None
        return self

    def __exit__(self, *exc):
        if self.proc is not None:
            time.sleep(0.15)
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
            self.fh.close()

    def summary(self):
        if self.proc is None or not self.path or not os.path.exists(self.path):
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unavailable"]}
        sm, mx, pw = [], [], []
        reasons = set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        with open(self.path) as f:
            for line in f:
                parts = [p.strip() for p in line.split(",")]
                if len(parts) < 9:
                    continue
                try:
                    sm.append(float(parts[1]))
                    mx.append(float(parts[2]))
                    pw.append(float(parts[3]))
                except ValueError:
                    continue
                for n, v in zip(names, parts[5:9]):
                    if v.lower() == "active":
                        reasons.add(n)
        os.unlink(self.path)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"]}
        # "under load": samples within the busiest part of the run
        top = sorted(sm)
        load = [s for s in sm if s >= 0.5 * top[-1]] or sm
        return {"sm_mhz": statistics.median(load), "sm_max_mhz": max(mx), "power_w_max": max(pw),
                "samples": len(sm), "reasons": sorted(reasons)}


# ---------------------------------------------------------------------------
# Algorithmic cost of each kernel, per launch (the roofline numerators)
# ---------------------------------------------------------------------------
def kernel_costs(wl, tables_bytes):
    """Algorithmic work per launch of each kernel: (bound, amount, unit).
    ``tables_bytes`` is one cos/sin table set (N L d/2 rotations x 8 bytes)."""
    d, N, k, T = wl.d, wl.n_experts, wl.k, wl.tokens
    R = T * k
    L = wl.stages
    xb = 2 if wl.dtype == "bf16" else 4
    ib = 2 if (wl.dtype == "bf16" and d >= 64) else 4  # Z and slot element size
    return {
        # GEMM: 2 R d^2 flops on the tensor cores
        "ternary_gemm_tc": ("tensor", 2.0 * R * d * d, "TFLOP/s"),
        # the whole expert in one kernel (pre-rotation, product, post-rotation,
        # gate): its contraction is the 2 R d^2 of the product
        "fused_expert": ("tensor", 2.0 * R * d * d, "TFLOP/s"),
        "ternary_gemm_simt": ("alu", 2.0 * R * d * d, "TFLOP/s"),
        # router product on the CUDA cores: 2 T N d flops
        "router_logits_simt": ("alu", 2.0 * T * N * d, "TFLOP/s"),
        # router on the tensor cores: the algorithmic 2 T N d (it issues 3x
        # that in bf16 MMAs for the exact split of the float32 gate weights)
        "router_tc": ("tensor", 2.0 * T * N * d, "TFLOP/s"),
        "router_split": ("hbm", N * d * 4 + 3 * N * d * 2, "GB/s"),
        # pre-rotation: x rows gathered (R rows) + X_rot written + the theta table
        "pre_rotate": ("hbm", R * d * xb + R * d * xb + tables_bytes, "GB/s"),
        # post-rotation: Z read + gated slots written + the phi table
        "post_rotate": ("hbm", R * d * ib + R * d * ib + tables_bytes, "GB/s"),
        "combine": ("hbm", R * d * ib + T * d * xb, "GB/s"),
        "rot_table": ("hbm", 2 * N * L * (d // 2) * 4 + 2 * tables_bytes, "GB/s"),
        "expand_base_bf16": ("hbm", d * d // 4 + 2 * d * d, "GB/s"),
        "router_topk": ("hbm", T * N * 4 + T * k * 8, "GB/s"),
    }


def alu_peak_tflops(sm_mhz):
    return SM_COUNT * FP32_LANES_PER_SM * 2 * sm_mhz * 1e6 / 1e12


# ---------------------------------------------------------------------------
# The CPU oracle as the baseline (host cores)
# ---------------------------------------------------------------------------
def oracle_expert_slice(inp, experts):
    """Oracle output for every routed row whose expert is in ``experts``
    (routing over all tokens, dense experts, per-expert products).
    Returns (rows evaluated, seconds)."""
    from oracle import bfmoe_oracle as O
    t0 = time.perf_counter()
    x = inp.x_f64()
    idx, gates, _, _ = O.route(x, inp.w_gate, inp.bias, inp.wl.k)
    flat = idx.reshape(-1)
    k = inp.wl.k
    y = np.zeros_like(x)
    rows = 0
    for e in experts:
        r = np.nonzero(flat == e)[0]
        if r.size == 0:
            continue
        We = O.expert_matrix(inp.w_base, inp.alpha, inp.theta[e], inp.phi[e])
        t, j = r // k, r % k
        np.add.at(y, t, gates[t, j][:, None] * (x[t] @ We.T))
        rows += r.size
    return rows, time.perf_counter() - t0


def cpu_cores():
    try:
        from threadpoolctl import threadpool_info
        th = max((i.get("num_threads", 1) for i in threadpool_info()), default=1)
    except Exception:  # noqa: BLE001
        th = os.cpu_count() or 1
    return th


def cpu_baseline(inp, frac_experts: float):
    N = inp.wl.n_experts
    n = max(1, int(round(N * frac_experts)))
    rows, sec = oracle_expert_slice(inp, range(n))
    return {"value": (rows / inp.wl.k) / sec, "unit": UNIT, "cores": cpu_cores(), "kind": "oracle",
            "sample": f"{inp.wl.describe()}: all tokens routed, rows of experts 0..{n - 1} "
                      f"({rows} rows = {rows / inp.wl.k:.0f} token-equivalents) formed densely and multiplied; "
                      f"{sec:.1f} s"}


def run_reference(args, wl):
    rank, world, _ = dist_env()
    if rank != 0:
        return 0
    inp = W.generate(wl, seed=0)
    N = wl.n_experts
    per = max(1, N // 16)
    times, units = [], []
    for step in range(args.warmup + args.steps):
        lo = (step * per) % N
        rows, sec = oracle_expert_slice(inp, range(lo, min(N, lo + per)))
        if step >= args.warmup:
            times.append(sec)
            units.append(rows / wl.k)
    total = sum(times)
    value = sum(units) / total
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * total / args.steps,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic", "config": workload_config(wl, "n/a (host)"),
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": cpu_cores(), "kind": "oracle",
                         "sample": f"each step: all {wl.tokens} tokens routed, rows of {per} consecutive "
                                   f"experts (of {N}) formed densely and multiplied"},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


def workload_config(wl, l2):
    return {"workload": wl.name, "d": wl.d, "n_experts": wl.n_experts, "k": wl.k, "tokens": wl.tokens,
            "x_dtype": wl.dtype, "routed_rows": wl.tokens * wl.k, "l2": l2, "parallelism": "token shards"}


# ---------------------------------------------------------------------------
# Our arm
# ---------------------------------------------------------------------------
def run_ours(args, wl):
    import torch
    import torch.distributed as dist

    rank, world, local = dist_env()
    if world != args.gpus:
        raise SystemExit(f"--gpus {args.gpus} but WORLD_SIZE={world}")
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=dev)

    from ternary_butterfly_experts_b200 import build as b
    if rank == 0:
        b.build()
    if world > 1:
        dist.barrier()
    import ternary_butterfly_experts_b200 as B
    from ternary_butterfly_experts_b200.shard import max_over_ranks, token_range

    peaks, peak_src = load_peaks()
    # weak scaling: rank r owns tokens [r*T, (r+1)*T) of a world*T batch
    a, _ = token_range(wl.tokens * world, rank, world)
    inp = W.generate(wl, seed=0, tokens=wl.tokens, token_offset=a)
    layer = B.Layer.from_host(inp.w_base, inp.alpha, inp.theta, inp.phi, device=dev)
    # the weight tables (cos/sin of the angles, the bf16 base) and the split
    # router weights are built once per layer load, outside the timed steps
    # (bfmoe_prepare_layer, bfmoe_prepare_gate); the step that rebuilds them
    # from the stored weights each time is reported apart
    layer.prepare()
    wg = torch.from_numpy(inp.w_gate).to(dev)
    layer.prepare_gate(wg)
    bias = None if inp.bias is None else torch.from_numpy(inp.bias).to(dev)
    x = inp.x.to(dev).contiguous()
    model = B.ButterflyMoE(layer, wg, bias, wl.k, wl.tokens, x.dtype)
    y = torch.empty_like(x)
    flush = torch.empty(512 * 1024 * 1024 // 4, dtype=torch.float32, device=dev)
    stream = torch.cuda.current_stream()

    def step():
        model(x, y=y)

    if args.ncu_run:
        # the launches a profiler captures: W warm-up steps, then K steps,
        # eager (no graph), nothing else
        for _ in range(args.warmup + args.steps):
            step()
        torch.cuda.synchronize()
        B.bfmoe_check_device_error()
        if rank == 0:
            print(json.dumps({"ncu_run": wl.name, "steps": args.steps, "warmup": args.warmup}), flush=True)
        if world > 1:
            dist.destroy_process_group()
        return 0

    def timed(n, fn, flush_l2=True):
        evs = []
        for _ in range(n):
            if flush_l2:
                flush.fill_(1.0)
            a = torch.cuda.Event(enable_timing=True)
            bb = torch.cuda.Event(enable_timing=True)
            a.record(stream)
            fn()
            bb.record(stream)
            evs.append((a, bb))
        torch.cuda.synchronize()
        return sum(a.elapsed_time(bb) for a, bb in evs)

    for _ in range(max(3, args.warmup)):
        step()
    B.bfmoe_check_device_error()
    torch.cuda.synchronize()
    n0 = B.bfmoe_launch_count()
    step()
    launches_per_step = B.bfmoe_launch_count() - n0
    torch.cuda.synchronize()

    # --- end to end through host buffers ----------------------------------------
    # (timed first, after its own warm-up: measured later in the process, after
    # the second-long device-only loops below, the same replays ran 5-45 %
    # slower, varying from one point to the next, so the other legs would
    # perturb it)
    # bfmoe_moe_forward_host: pinned host tokens in, pinned host outputs out,
    # the copies overlapped with the work in token chunks; the call is
    # captured once as a CUDA graph (copies included) and replayed per step
    x_host = inp.x.pin_memory()
    y_host = torch.empty(x.shape, dtype=x.dtype).pin_memory()
    model.forward_host(x_host, y_host)  # creates the copy streams before capture
    torch.cuda.synchronize()
    host_graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(host_graph):
        model.forward_host(x_host, y_host)

    for _ in range(max(3, args.warmup)):
        host_graph.replay()
    e2e_ms = timed(args.steps, host_graph.replay)
    e2e_ms = max_over_ranks(e2e_ms)
    for _ in range(max(3, args.warmup)):
        model.forward_host(x_host, y_host)
    e2e_eager_ms = timed(args.steps, lambda: model.forward_host(x_host, y_host))
    e2e_eager_ms = max_over_ranks(e2e_eager_ms)
    B.bfmoe_check_device_error()

    # router + forward captured once as a CUDA graph; each step is one replay
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        step()
    graph.replay()
    torch.cuda.synchronize()
    B.bfmoe_check_device_error()

    # --- timed region ---------------------------------------------------------
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    with ClockSampler(physical_gpu_index(local)) as clocks:
        total_ms = timed(args.steps, graph.replay)
    launches = launches_per_step * args.steps
    torch.cuda.synchronize()
    # sustained window: >= 1 s of timed graph replays (L2 flushed between
    # them, outside the timed intervals), with its own clock samples
    step_s = max(1e-6, total_ms / args.steps / 1e3)
    sus_n = max(args.steps, int(math.ceil(1.0 / step_s)))
    with ClockSampler(physical_gpu_index(local)) as sus_clocks:
        sus_ms = timed(sus_n, graph.replay)
    sus_ms = max_over_ranks(sus_ms)
    eager_ms = timed(args.steps, step)
    # the same step with the weight tables and the router split rebuilt in it
    layer.unprepare()
    layer.unprepare_gate()
    step()  # first unprepared call creates the side stream before capture
    torch.cuda.synchronize()
    graph_rt = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph_rt):
        step()
    graph_rt.replay()
    torch.cuda.synchronize()
    rt_ms = max_over_ranks(timed(args.steps, graph_rt.replay))
    del graph_rt
    layer.prepare()
    layer.prepare_gate(wg)
    if world > 1:
        dist.barrier()
    total_ms = max_over_ranks(total_ms)
    B.bfmoe_check_device_error()

    # --- per-kernel device times (same steps again, each launch bracketed) ------
    B.bfmoe_profile_enable(True)
    prof_ms = timed(args.steps, step)
    kt = B.bfmoe_profile_collect()
    B.bfmoe_profile_enable(False)


    # --- decode batches: router + the add-only forward, T = 64 -------------------
    dec_T = min(64, wl.tokens)
    dec = B.ButterflyMoE(layer, wg, bias, wl.k, dec_T, x.dtype)
    xd = x[:dec_T].contiguous()
    yd = torch.empty_like(xd)
    for _ in range(max(3, args.warmup)):
        dec.decode(xd, y=yd)
    torch.cuda.synchronize()
    dec_graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(dec_graph):
        dec.decode(xd, y=yd)
    dec_graph.replay()
    torch.cuda.synchronize()
    dec_steps = 200
    dec_ms = timed(dec_steps, dec_graph.replay, flush_l2=False)
    B.bfmoe_profile_enable(True)
    timed(20, lambda: dec.decode(xd, y=yd), flush_l2=False)
    dkt = B.bfmoe_profile_collect()
    B.bfmoe_profile_enable(False)
    B.bfmoe_check_device_error()

    # --- backward: dx, both angle sets, the base (straight-through), alpha, W_g, b
    routing = (model.idx[:wl.tokens], model.gates[:wl.tokens], model.counts, model.offsets,
               model.rows[:wl.tokens * wl.k])
    g = torch.Generator(device=dev)
    g.manual_seed(1)
    gy = torch.randn(x.shape, dtype=torch.float32, device=dev, generator=g)
    bw_ws = torch.empty(max(B.bfmoe_backward_workspace_size(wl.d, wl.n_experts, wl.tokens, wl.k), 256),
                        dtype=torch.uint8, device=dev)

    def backward():
        B.bfmoe_backward(layer, x, wl.k, wg, routing, gy, bias_grad=bias is not None, ws=bw_ws)

    for _ in range(2):
        backward()
    torch.cuda.synchronize()
    bw_steps = 3
    bw_ms = timed(bw_steps, backward)
    B.bfmoe_check_device_error()

    if rank == 0:
        clk = clocks.summary()
        T = wl.tokens
        value = T * world * args.steps / (total_ms / 1e3)
        L = wl.stages
        costs = kernel_costs(wl, wl.n_experts * L * (wl.d // 2) * 8)
        kernels = {}
        for name, (n, ms) in kt.items():
            entry = {"launches": n, "total_ms": ms, "share": ms / max(1e-9, sum(v[1] for v in kt.values())),
                     "avg_us": 1e3 * ms / n}
            kernels[name] = entry
        # the dominant kernel of the critical path: the table build runs on the
        # side stream, overlapped with the router
        main = {k: v for k, v in kt.items() if k not in SIDE_STREAM_KERNELS} or kt
        dom = max(main.items(), key=lambda kv: kv[1][1])[0]
        # a contraction timed inside a long step runs under the power cap:
        # its peak is then the sustained GEMM figure, else the burst one
        long_step = total_ms / args.steps > 1.0
        roof = roofline_entry(dom, kt[dom], costs, peaks, clk, workload=wl.name, sustained=long_step)
        roof["algorithmic"] = ("2 R d^2 flops of the ternary product (R = T k routed rows); the fused "
                               "kernel's inputs and outputs are the path's own bytes") \
            if roof["bound"] == "tensor" else "bytes of the kernel's inputs and outputs"
        if dom == "fused_expert":
            # the same kernel seen from its CUDA-core work: two butterflies of
            # L stages of d/2 rotations (4 multiplies, 2 adds) per routed row
            rot_flops = 6.0 * T * wl.k * wl.d * L
            avg_s = kt[dom][1] / kt[dom][0] / 1e3
            fp32_peak = alu_peak_tflops(clk.get("sm_mhz") or 1965.0)
            roof["rotation_view"] = {"bound": "alu", "flops_per_launch": rot_flops,
                                     "achieved": rot_flops / avg_s / 1e12, "peak": fp32_peak, "unit": "TFLOP/s",
                                     "frac": rot_flops / avg_s / 1e12 / fp32_peak,
                                     "peak_source": "fp32 FMA lanes x 2 x median SM clock under load"}
        as_built = as_built_bytes(wl)
        flops = 2.0 * T * wl.k * wl.d ** 2
        bytes_alg = algorithmic_bytes(wl)
        t_roof = max(flops / (peaks["bf16_tflops"] * 1e12), bytes_alg / (peaks["hbm_gbs"] * 1e9))
        line = {
            "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": total_ms / args.steps, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": wl.dtype, "data": "synthetic",
            "config": workload_config(wl, "flushed between steps (512 MiB write, outside the timed intervals)"),
            "roofline": roof,
            "as_built_traffic": as_built,
            "path_roofline": {"time_us": t_roof * 1e6, "achieved_us": 1e3 * total_ms / args.steps,
                              "frac": t_roof / (total_ms / args.steps / 1e3),
                              "formula": "max(2 T k d^2 / bf16 peak, algorithmic bytes / HBM BW)",
                              "peak_source": peak_src},
            "kernels": kernels,
            "profiled_pass_ms_per_step": prof_ms / args.steps,
            "eager_ms_per_step": eager_ms / args.steps,
            "timing": "CUDA-graph replay of router + forward per step (captured once); "
                      "kernels timed individually in a separate eager pass",
            "cpu_baseline": None,
            "e2e": {"value": T * world * args.steps / (e2e_ms / 1e3), "unit": UNIT,
                    "h2d_bytes_per_step": int(x_host.numel() * x_host.element_size()),
                    "d2h_bytes_per_step": int(y_host.numel() * y_host.element_size()),
                    "call": "bfmoe_moe_forward_host (pinned host buffers, copies overlapped in token chunks), "
                            "captured once as a CUDA graph and replayed per step; timed first, after its own "
                            "warm-up, before the device-only legs",
                    "eager_value": T * world * args.steps / (e2e_eager_ms / 1e3)},
            "gpu_launches": int(launches),
            "weight_tables": "prepared once per layer load (bfmoe_prepare_layer, bfmoe_prepare_gate), "
                             "outside the timed steps",
            "tables_rebuilt_per_step": {"ms_per_step": rt_ms / args.steps,
                                        "value": T * world * args.steps / (rt_ms / 1e3),
                                        "note": "the cos/sin tables, the bf16 base (on a side stream) and the "
                                                "router's W_g split rebuilt from the stored weights inside every step"},
            "sustained": {"steps": sus_n, "timed_seconds": sus_ms / 1e3, "ms_per_step": sus_ms / sus_n,
                          "value": T * world * sus_n / (sus_ms / 1e3), "clocks": sus_clocks.summary()},
            "backward": {"call": "bfmoe_backward (dx, dtheta, dphi, straight-through dW_base, dalpha, dW_g, db) "
                                 "on the step's routing, eager, L2 flushed", "steps": bw_steps,
                         "ms_per_step": bw_ms / bw_steps, "tokens_per_s": T * bw_steps / (bw_ms / 1e3)},
            "decode": {"tokens": dec_T, "call": "router (bfmoe_router_topk, no buckets) + bfmoe_decode_forward (add-only "
                       "ternary product, float32 inside), CUDA-graph replays, weights L2-resident",
                       "us_per_step": 1e3 * dec_ms / dec_steps,
                       "tokens_per_s": dec_T * dec_steps / (dec_ms / 1e3),
                       "kernels_us": {n: 1e3 * ms / c for n, (c, ms) in dkt.items()}},
            "clocks": clk,
        }
        if world == 1 and not args.no_cpu_baseline:
            line["cpu_baseline"] = cpu_baseline(inp, args.cpu_fraction)
        print(json.dumps(line), flush=True)
    del graph, host_graph, dec_graph
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    return 0


def as_built_bytes(wl):
    """Memory traffic the built pipeline adds per step on top of the
    algorithmic bytes (not counted in any roofline fraction)."""
    d, N, k, T = wl.d, wl.n_experts, wl.k, wl.tokens
    L = wl.stages
    R = T * k
    xb = 2 if wl.dtype == "bf16" else 4
    fused = wl.dtype == "bf16" and 64 <= d <= 512
    out = {
        "router_logits_f32": T * N * 4,                     # written for the fix-up of undecided tokens
        "router_weight_split_bf16": 3 * N * d * 2,          # written, then read by the tensor-core router
        "x_gather_rereads": (k - 1) * T * d * xb,           # each token's row is read once per slot
        "weight_tables": 2 * N * L * (d // 2) * 8 * 2,      # cos/sin quads written and read per step
        "base_bf16_copy": 2 * d * d * 2,                    # the expanded base, written and read
        "slot_buffer": 2 * R * d * (2 if fused else 4),     # gated rows written, then summed by the combine
    }
    if not fused:
        out["x_rot_round_trip"] = 2 * R * d * (2 if wl.dtype == "bf16" else 4)
        out["z_round_trip"] = 2 * R * d * (2 if wl.dtype == "bf16" else 4)
    out["total"] = sum(out.values())
    return out


def algorithmic_bytes(wl):
    """x read once, y written once, packed base, angles, router weights and
    bias, routing outputs."""
    d, N, k, T = wl.d, wl.n_experts, wl.k, wl.tokens
    xb = 2 if wl.dtype == "bf16" else 4
    return (2 * T * d * xb + d * d // 4 + 2 * N * wl.stages * (d // 2) * 4 + N * d * 4 + N * 4
            + T * k * 8)


# Launch names of the library -> kernel names in the ncu summaries.
SIDE_STREAM_KERNELS = {"rot_table"}

NCU_KERNEL = {"fused_expert": "fused_expert_kernel", "post_rotate": "post_rotate_fast_kernel", "pre_rotate": "pre_rotate_fast_kernel",
              "ternary_gemm_tc": "ternary_gemm_tc_kernel", "router_tc": "router_tc_kernel",
              "combine": "combine_kernel", "rot_table": "rot_quads_kernel"}


def kernel_sources_hash() -> str:
    """sha256 over the library's CUDA sources under ROOT (sorted by name)."""
    from ternary_butterfly_experts_b200.ncu_summary import kernel_sources_hash as h
    return h(os.path.join(ROOT, "ternary_butterfly_experts_b200", "csrc"))


def profiled_traffic(name, workload):
    """DRAM bytes (read + write) of one launch of kernel `name`, from the
    committed ncu summary (profiles/ncu_*_<workload>.json, written by
    ternary_butterfly_experts_b200.ncu_summary), or None when there is none or
    the kernel sources have changed since it was taken."""
    import glob
    kname = NCU_KERNEL.get(name)
    if kname is None:
        return None
    src_hash = kernel_sources_hash()
    for path in sorted(glob.glob(os.path.join(ROOT, "profiles", f"ncu_*_{workload}.json"))):
        with open(path) as f:
            js = json.load(f)
        if js.get("kernel_sources_sha256") != src_hash:
            continue
        for kn, e in js.get("kernels", {}).items():
            if kn.split("<")[0] == kname and "dram_bytes_per_launch" in e:
                return float(e["dram_bytes_per_launch"])
    return None


def roofline_entry(name, kt_entry, costs, peaks, clk, workload=None, sustained=False):
    n, ms = kt_entry
    avg_s = ms / n / 1e3
    bound, work, unit = costs.get(name, ("hbm", float("nan"), "GB/s"))
    if bound == "tensor":
        achieved = work / avg_s / 1e12
        if sustained and peaks.get("bf16_tflops_sustained"):
            peak = peaks["bf16_tflops_sustained"]
            src = "bf16_tflops_sustained (measured; the kernel runs inside a step of more than 1 ms)"
        else:
            peak = peaks["bf16_tflops"]
            src = "bf16_tflops (measured burst)"
    elif bound == "alu":
        achieved = work / avg_s / 1e12
        mhz = peaks.get("sm_max_mhz", 1965.0)
        peak = alu_peak_tflops(mhz)
        src = f"fp32 FMA: {SM_COUNT} SMs x {FP32_LANES_PER_SM} lanes x 2 x {mhz:.0f} MHz"
    else:
        achieved = work / avg_s / 1e9
        peak = peaks["hbm_gbs"]
        src = "hbm_gbs (measured copy)"
    traffic = profiled_traffic(name, workload) if workload else None
    return {"kernel": name, "bound": bound, "achieved": achieved, "peak": peak, "unit": unit,
            "frac": achieved / peak, "traffic": traffic, "avg_launch_us": avg_s * 1e6,
            "work_per_launch": work, "peak_source": src,
            "traffic_source": "ncu dram__bytes_read.sum + dram__bytes_write.sum, first launch "
                              "(profiles/ncu_*.json of the current kernel sources)"
            if traffic is not None else "no ncu summary taken from the current kernel sources"}


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--workload", default=W.HEADLINE, choices=sorted(W.WORKLOADS))
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--ncu-run", action="store_true",
                    help="run warm-up + steps eagerly and exit (the command profiled under ncu)")
    ap.add_argument("--cpu-fraction", type=float, default=1.0,
                    help="fraction of the experts whose rows the CPU baseline evaluates")
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3
    wl = W.WORKLOADS[args.workload]
    if args.impl == "reference":
        return run_reference(args, wl)
    return run_ours(args, wl)


if __name__ == "__main__":
    sys.exit(main())
