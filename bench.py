"""Benchmark of the W4 + per-token-gated EC linear layer on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference] [--workload NAME]

A step is one pass of the whole hot path over one batch of the workload: for the default
workload (decode q/o-projection, N = K = 4096, EC rank 64, 1% outlier channels x20) that is
one spear_w4ec_gemm call for each decode batch M in {1, 4, 16}; each call runs the EC
pre-pass and the weight-streaming GEMM.  Packing runs once, before timing.

value   = algorithmic bytes (packed W4 + s/z + A + B + w_g + x + y) / device time, GB/s,
          inputs resident in HBM; K steps are captured in a CUDA graph and replayed, timed
          with CUDA events; weights rotate over copies larger than 2x L2.
e2e     = same metric through the Python API with pinned host x and y: every step copies x
          host->device and y device->host inside the timed region.
roofline= the layer call at the largest decode batch, against the measured HBM copy peak.
cpu_baseline / --impl reference = the CPU oracle timed on this host's cores on a bounded
          sample of the same workload.

Multi-GPU (torchrun): independent replicas, one per GPU (no data-path collective); the
timed region is bracketed by barriers and the max over ranks is reported.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

WORKLOADS = {
    # name: (config index, batches, kind)
    "decode-qo": (1, [1, 4, 16], "decode"),
    "decode-mlp": (2, [1, 8, 32, 64], "decode"),
    "prefill": (3, [2048], "prefill"),
}
# Plan sweeps only (--sweep): the four linear shapes of the 16-layer model (rank-32 compensator).
SWEEP_ONLY = {"sweep-1b": (4, [1, 16, 256, 4096])}
L2_BYTES = 126 * 1024 * 1024


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--workload", default="decode-qo", choices=sorted(WORKLOADS) + sorted(SWEEP_ONLY))
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-prefill", action="store_true", help="skip the secondary prefill measurement")
    ap.add_argument("--no-detail", action="store_true",
                    help="skip the secondary decode-mlp and 16-layer model figures of the default run")
    ap.add_argument("--cpu-seconds", type=float, default=10.0)
    ap.add_argument("--sweep", action="store_true",
                    help="time every valid decode tiling for the workload's batches and print a table")
    ap.add_argument("--batches", default="", metavar="M1,M2,..",
                    help="with --sweep: time only these batch sizes of the workload")
    ap.add_argument("--once", type=int, default=0, metavar="M",
                    help="run 5 layer calls of the workload with M tokens and exit (for profilers)")
    ap.add_argument("--no-ec", action="store_true", help="with --once: the plain W4 layer")
    ap.add_argument("--linear", type=int, default=0, choices=[0, 1, 2, 3],
                    help="with --once --workload sweep-1b: which linear of the model's layer 0")
    ap.add_argument("--plan", default="", metavar="KERNEL,TILE_N,TILE_M,SPLIT_K,FLAGS",
                    help="with --once: this plan (checked by spear_plan_update) instead of the planner's")
    ap.add_argument("--model-sweep", action="store_true",
                    help="the 16-layer sweep workload (hidden 2048, MLP 8192, EC r=32 on layers 0, 1, 7, 15): "
                         "all 64 linears of one pass per batch size, with the dispatcher's plans")
    ap.add_argument("--slo-check", action="store_true",
                    help="SLO-constrained prefill chunk picker on the 16-layer model: picked chunk, predicted "
                         "and measured step time per ITL target")
    ap.add_argument("--grouped-compare", action="store_true",
                    help="per-channel vs group-wise (128) scales on the decode-qo layer, EC on and off")
    ap.add_argument("--gate-compare", action="store_true",
                    help="time the layer with the scalar gate and with the bottleneck-MLP gate (H=16) on "
                         "decode-qo M=16 and the prefill layer")
    ap.add_argument("--svd-demo", action="store_true",
                    help="static SVD-initialised compensator on the workload's layer: share of the 4-bit "
                         "output error removed and time per call, for several ranks")
    return ap.parse_args()


def measured_traffic(kernel: str):
    """DRAM bytes per launch of `kernel` from the committed ncu summary, or None when the kernel's
    source has changed since those counters were taken."""
    import hashlib
    path = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(path):
        return None
    entry = json.load(open(path)).get(kernel)
    if not entry:
        return None
    src = os.path.join(ROOT, entry["source"])
    if not os.path.exists(src) or hashlib.sha256(open(src, "rb").read()).hexdigest()[:16] != entry["source_sha256_16"]:
        return None
    return {"bytes_per_launch": entry["dram_bytes_per_launch"], "workload": entry["workload"]}


def layer_bytes(M, N, K, r):
    w = N * K // 2 + 4 * N
    ec = (2 * K * r + 2 * r * N + 2 * K) if r else 0
    return w + ec + 2 * M * K + 2 * M * N


def layer_flops(M, N, K, r):
    f = 2 * M * N * K
    if r:
        f += 2 * M * K * r + 2 * M * r * N + 2 * M * K
    return f


# ----------------------------------------------------------------------------- clocks

class ClockSampler:
    """nvidia-smi samples (every 100 ms, timestamped) for the whole run; summary() keeps the ones
    that fall inside a given wall-clock window."""
    FIELDS = ("timestamp,index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")
    REASONS = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]

    def __init__(self, device_index: int):
        self.dev = device_index
        self.proc = None
        self.lines = []

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.dev), f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "100"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None
        time.sleep(0.5)  # let the first samples arrive
        return self

    def stop(self):
        if self.proc is not None:
            self.proc.terminate()
            try:
                out, _ = self.proc.communicate(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
                out, _ = self.proc.communicate()
            self.lines = [ln for ln in out.splitlines() if ln.strip()]
            self.proc = None

    def samples(self):
        import datetime
        out = []
        for ln in self.lines:
            parts = [p.strip() for p in ln.split(",")]
            if len(parts) < 10:
                continue
            try:
                ts = datetime.datetime.strptime(parts[0], "%Y/%m/%d %H:%M:%S.%f").timestamp()
                sm, mx = float(parts[2]), float(parts[3])
            except ValueError:
                continue
            active = [nm for nm, v in zip(self.REASONS, parts[6:10]) if v.lower().startswith("active")]
            out.append((ts, sm, mx, active))
        return out

    def summary(self, t0, t1, where):
        sel = [s for s in self.samples() if t0 <= s[0] <= t1]
        if not sel:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0, "window": where}
        reasons = sorted({r for s in sel for r in s[3]})
        return {"sm_mhz": statistics.median(s[1] for s in sel), "sm_max_mhz": max(s[2] for s in sel),
                "reasons": reasons, "samples": len(sel), "window": where}


# ----------------------------------------------------------------------------- replicas

def max_over_ranks(dist, seconds: float, device) -> float:
    """The slowest rank's time: every rank gets the max (all-reduce MAX)."""
    import torch
    t = torch.tensor([seconds], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def replica_throughput(units_per_rank: float, world: int, max_seconds: float) -> float:
    """Whole-job throughput of `world` independent replicas timed by the slowest one."""
    return units_per_rank * world / max_seconds


# ----------------------------------------------------------------------------- CPU oracle

def oracle_sample(widx, seconds, M_list):
    """Time the CPU oracle on the workload's batches, repeated for about `seconds`."""
    import oracle
    from synthetic import config_layers
    cfg, batches, kind = WORKLOADS[widx]
    L = config_layers(cfg, M=max(batches))[0]
    packed, s, z = oracle.pack_w4(L.W)
    if kind == "prefill":
        M_list = [64]          # a 64-token slice of the 2048-token batch (rows are independent)
    total_bytes = total_flops = 0
    reps = 0
    t0 = time.perf_counter()
    while True:
        for M in M_list:
            oracle.w4ec_gemm(L.x(M), packed, s, z, L.A_bits, L.B_bits, L.wg_bits, L.b_g)
            total_bytes += layer_bytes(M, L.N, L.K, L.rank)
            total_flops += layer_flops(M, L.N, L.K, L.rank)
        reps += 1
        if time.perf_counter() - t0 >= seconds:
            break
    dt = time.perf_counter() - t0
    return {"bytes": total_bytes, "flops": total_flops, "seconds": dt, "reps": reps, "M": M_list,
            "cores": oracle.num_threads()}


def cpu_baseline_obj(widx, seconds):
    cfg, batches, kind = WORKLOADS[widx]
    r = oracle_sample(widx, seconds, batches)
    if kind == "prefill":
        val, unit = r["flops"] / r["seconds"] / 1e12, "TFLOP/s"
    else:
        val, unit = r["bytes"] / r["seconds"] / 1e9, "GB/s"
    return {"value": val, "unit": unit, "cores": r["cores"], "kind": "oracle",
            "sample": f"{r['reps']} passes over M={r['M']} of the {widx} layer, fp64 C oracle, "
                      f"{r['seconds']:.1f} s"}


# ----------------------------------------------------------------------------- GPU arm

def make_device_layer(torch, spear, L, copies):
    dev = torch.device("cuda")
    W = torch.from_numpy(L.W).to(dev)
    packed, scale, zero = spear.spear_pack_w4(W)
    del W
    bf = lambda a: torch.from_numpy(a.view(np.int16)).to(dev).view(torch.bfloat16)
    A, B, wg = bf(L.A_bits), bf(L.B_bits), bf(L.wg_bits)
    sets = []
    for c in range(copies):
        if c == 0:
            sets.append((packed, scale, zero, A, B, wg))
        else:
            sets.append(tuple(t.clone() for t in (packed, scale, zero, A, B, wg)))
    return sets


def run_ours(args, rank, world, torch, dist):
    import w4_gemm_error_channel_b200 as spear
    from synthetic import config_layers

    cfg, batches, kind = WORKLOADS[args.workload]
    L = config_layers(cfg, M=max(batches))[0]
    N, K, r = L.N, L.K, L.rank
    per_set = layer_bytes(max(batches), N, K, r)
    copies = max(2, int(np.ceil(2 * L2_BYTES / per_set)) + 1)
    if kind == "prefill":
        copies = max(2, int(np.ceil(2 * L2_BYTES / (N * K // 2 + 2 * max(batches) * K))))
    sets = make_device_layer(torch, spear, L, copies)
    dev = torch.device("cuda")
    xs = {M: torch.from_numpy(L.x(M).view(np.int16)).to(dev).view(torch.bfloat16) for M in batches}
    ys = {M: torch.empty((M, N), dtype=torch.bfloat16, device=dev) for M in batches}
    # Both code orders at hand (the tile order is made once, like the packing): each batch size is
    # planned on the order measured faster for it.
    tileable = kind == "decode" and N % 128 == 0 and K % 128 == 0
    tiled = [spear.spear_tile_w4(p) for (p, *_) in sets] if tileable else None
    fmts = spear.SPEAR_W4_ROWS | (spear.SPEAR_W4_TILES if tileable else 0)
    plans = {M: spear.spear_gemm_plan_formats(M, N, K, r, fmts) for M in batches}
    plans_no_ec = {M: spear.spear_gemm_plan_formats(M, N, K, 0, fmts) for M in batches}
    ws = spear.alloc_workspace(max(p.workspace_bytes for p in list(plans.values()) + list(plans_no_ec.values())))
    stream = torch.cuda.Stream()
    calls_per_step = len(batches)

    def codes(i, plan):
        return tiled[i] if plan.flags & spear.SPEAR_PLAN_W4_TILES else sets[i][0]

    def step_calls(step_idx, use_ec=True):
        for j, M in enumerate(batches):
            i = (step_idx * calls_per_step + j) % copies
            p, s, z, A, B, wg = sets[i]
            ec = spear.EC(A, B, wg, L.b_g) if use_ec else None
            spear.spear_w4ec_gemm(xs[M], codes(i, plans[M]), s, z, ec, y=ys[M], workspace=ws, plan=plans[M],
                                  stream=stream)

    def graph_of(n_steps, use_ec=True, only_M=None):
        g = torch.cuda.CUDAGraph()
        with torch.cuda.stream(stream):
            # warm the path (library attributes, first launches) before capture
            step_calls(0, use_ec)
            stream.synchronize()
            with torch.cuda.graph(g, stream=stream):
                for i in range(n_steps):
                    if only_M is None:
                        step_calls(i, use_ec)
                    else:
                        p, s, z, A, B, wg = sets[i % copies]
                        ec = spear.EC(A, B, wg, L.b_g) if use_ec else None
                        pl = plans[only_M] if use_ec else plans_no_ec[only_M]
                        spear.spear_w4ec_gemm(xs[only_M], codes(i % copies, pl), s, z, ec, y=ys[only_M],
                                              workspace=ws, plan=pl, stream=stream)
        return g

    def time_graph(g, reps=1):
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        with torch.cuda.stream(stream):
            e0.record(stream)
            for _ in range(reps):
                g.replay()
            e1.record(stream)
        e1.synchronize()
        return e0.elapsed_time(e1) / 1e3

    # Warm-up: W untimed steps (eager), then the graph once.
    for i in range(args.warmup):
        with torch.cuda.stream(stream):
            step_calls(i)
    stream.synchronize()
    g_main = graph_of(args.steps)
    with torch.cuda.stream(stream):
        g_main.replay()
    torch.cuda.synchronize()

    # Timed region: barrier + sync on both sides, K steps, max over ranks.
    clk = ClockSampler(torch.cuda.current_device()).start()
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    w0 = time.time()
    t_main = time_graph(g_main)
    torch.cuda.synchronize()
    w1 = time.time()
    if world > 1:
        t_main = max_over_ranks(dist, t_main, dev)
        dist.barrier()
    # The timed region is often shorter than the 100 ms sampling period: then the clocks are
    # read during an untimed soak of the same graph right after it.
    soak0 = time.time()
    while time.time() - soak0 < 1.5:
        time_graph(g_main)
    soak1 = time.time()
    time.sleep(0.3)
    clk.stop()
    clocks = clk.summary(w0, w1, "timed region")
    if clocks["samples"] < 3:
        clocks = clk.summary(soak0, soak1, "soak of the timed graph right after the timed region")

    step_bytes = sum(layer_bytes(M, N, K, r) for M in batches)
    step_flops = sum(layer_flops(M, N, K, r) for M in batches)

    # Per-batch timings (EC on and off) for the roofline and the EC overhead.
    per_m = {}
    n_sub = 64 if kind == "decode" else 8
    for M in batches:
        g_on = graph_of(n_sub, True, M)
        g_off = graph_of(n_sub, False, M)
        time_graph(g_on)
        time_graph(g_off)
        t_on = min(time_graph(g_on) for _ in range(3)) / n_sub
        t_off = min(time_graph(g_off) for _ in range(3)) / n_sub
        b_on, b_off = layer_bytes(M, N, K, r), layer_bytes(M, N, K, 0)
        per_m[M] = {"us": t_on * 1e6, "us_no_ec": t_off * 1e6, "GBps": b_on / t_on / 1e9,
                    "GBps_no_ec": b_off / t_off / 1e9, "TFLOPs": layer_flops(M, N, K, r) / t_on / 1e12,
                    "ec_overhead": t_on / t_off - 1.0, "ec_byte_floor": b_on / b_off - 1.0,
                    "plan": {"kernel": kernel_name(spear, plans[M]), "tile_n": plans[M].tile_n,
                             "split_k": plans[M].split_k, "tile_m": plans[M].tile_m, "flags": plans[M].flags},
                    "plan_no_ec": {"kernel": kernel_name(spear, plans_no_ec[M]), "split_k": plans_no_ec[M].split_k,
                                   "tile_m": plans_no_ec[M].tile_m, "flags": plans_no_ec[M].flags}}
        del g_on, g_off

    # e2e through the public API with pinned host buffers: a step's activations travel in one
    # host-to-device copy and its outputs in one device-to-host copy (one buffer each, a view per
    # call), as a serving loop batches them.
    tot_m = sum(batches)
    hx_all = torch.empty((tot_m * K,), dtype=torch.bfloat16).pin_memory()
    hy_all = torch.empty((tot_m * N,), dtype=torch.bfloat16).pin_memory()
    dx_all = torch.empty((tot_m * K,), dtype=torch.bfloat16, device=dev)
    dy_all = torch.empty((tot_m * N,), dtype=torch.bfloat16, device=dev)
    ex, ey, off = {}, {}, 0
    for M in batches:
        hx_all[off * K:(off + M) * K].copy_(torch.from_numpy(L.x(M).view(np.int16)).view(torch.bfloat16).reshape(-1))
        ex[M] = dx_all[off * K:(off + M) * K].view(M, K)
        ey[M] = dy_all[off * N:(off + M) * N].view(M, N)
        off += M
    e2e_steps = max(3, min(args.steps, 20))

    # The public API a serving loop uses: each weight set bound once as a W4ECLayer.
    e2e_layers = [spear.W4ECLayer(p, s, z, spear.EC(A, B, wg, L.b_g), tiled=tiled[i] if tiled else None)
                  for i, (p, s, z, A, B, wg) in enumerate(sets)]
    for lay in e2e_layers:
        for M in batches:
            lay.plan(M)

    def e2e_step(i):
        dx_all.copy_(hx_all, non_blocking=True)
        for j, M in enumerate(batches):
            lay = e2e_layers[(i * calls_per_step + j) % copies]
            lay(ex[M], y=ey[M], stream=stream)
        hy_all.copy_(dy_all, non_blocking=True)

    with torch.cuda.stream(stream):
        for i in range(2):
            e2e_step(i)
    stream.synchronize()
    if world > 1:
        dist.barrier()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with torch.cuda.stream(stream):
        e0.record(stream)
        for i in range(e2e_steps):
            e2e_step(i)
        e1.record(stream)
    e1.synchronize()
    t_e2e = e0.elapsed_time(e1) / 1e3
    if world > 1:
        t_e2e = max_over_ranks(dist, t_e2e, dev)

    import json as _json
    peaks = {}
    pk_path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(pk_path):
        peaks = _json.load(open(pk_path))
    hbm_peak = peaks.get("hbm_gbs", 6650.0)
    tc_peak = peaks.get("bf16_tflops", 1590.0)
    peak_src = "measured" if peaks else "fallback"

    if kind == "decode":
        metric_val = replica_throughput(step_bytes * args.steps, world, t_main) / 1e9
        unit = "GB/s"
        e2e_val = replica_throughput(step_bytes * e2e_steps, world, t_e2e) / 1e9
        Mr = max(b for b in batches if b <= 16) if any(b <= 16 for b in batches) else max(batches)
        tr = measured_traffic("w4ec_decode_kernel") if (plans[Mr].kernel_id == spear.SPEAR_KERNEL_SPLITK and
                                                        args.workload == "decode-qo" and Mr == 16) else None
        rl = {"bound": "hbm", "achieved": per_m[Mr]["GBps"], "peak": hbm_peak, "unit": "GB/s",
              "frac": per_m[Mr]["GBps"] / hbm_peak, "traffic": tr["bytes_per_launch"] if tr else None,
              "kernel": f"spear_w4ec_gemm M={Mr} ({kernel_name(spear, plans[Mr])}, EC fused into the weight stream)",
              "peak_source": f"{peak_src} hbm_gbs (copy)", "algorithmic_bytes": layer_bytes(Mr, N, K, r)}
    else:
        metric_val = replica_throughput(step_flops * args.steps, world, t_main) / 1e12
        unit = "TFLOP/s"
        e2e_val = replica_throughput(step_flops * e2e_steps, world, t_e2e) / 1e12
        M0 = batches[0]
        ach = per_m[M0]["TFLOPs"]
        tr = measured_traffic("w4_tc05_kernel") if args.workload == "prefill" else None
        rl = {"bound": "tensor", "achieved": ach, "peak": tc_peak, "unit": "TFLOP/s", "frac": ach / tc_peak,
              "traffic": tr["bytes_per_launch"] if tr else None, "kernel": f"spear_w4ec_gemm M={M0} (w4_tc05_kernel)",
              "peak_source": f"{peak_src} bf16_tflops (burst)", "algorithmic_flops": layer_flops(M0, N, K, r)}

    out = {
        "metric": "W4+gated-EC GEMM: decode GB/s and prefill TFLOP/s vs B200 roofline, 1 GPU",
        "value": metric_val, "unit": unit, "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": t_main / args.steps * 1e3, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": {"workload": f"{args.workload}: M in {batches}, N={N}, K={K}, EC rank {r}",
                   "l2": f"weights rotate over {copies} copies ({copies * per_set / 2**20:.0f} MiB > 2x L2)",
                   "parallelism": f"replicas x{world}", "timing": "CUDA graph of K steps, CUDA events"},
        "e2e": {"value": e2e_val, "unit": unit,
                "h2d_bytes_per_step": sum(2 * M * K for M in batches),
                "d2h_bytes_per_step": sum(2 * M * N for M in batches)},
        "gpu_launches": args.steps * sum(launches_per_call(spear, plans[M], M, r > 0) for M in batches),
        "roofline": rl,
        "clocks": clocks,
        "detail": {str(M): v for M, v in per_m.items()},
    }
    return out


def prefill_summary(torch, spear):
    """Secondary number: the prefill workload's TFLOP/s (M=2048, N=4096, K=14336, r=128)."""
    from synthetic import config_layers
    L = config_layers(3)[0]
    M, N, K, r = 2048, L.N, L.K, L.rank
    dev = torch.device("cuda")
    sets = make_device_layer(torch, spear, L, 3)
    x = torch.from_numpy(L.x(M).view(np.int16)).to(dev).view(torch.bfloat16)
    y = torch.empty((M, N), dtype=torch.bfloat16, device=dev)
    res = {}
    for variant in ("ec", "no_ec", "ec_semifused"):
        use_ec = variant != "no_ec"
        plan = spear.spear_gemm_plan(M, N, K, r if use_ec else 0)
        if variant == "ec_semifused":
            # The same tiling with the compensator as its own kernels beside the GEMM.
            plan.kernel_id, plan.split_k, plan.flags = spear.SPEAR_KERNEL_TC05, 1, spear.SPEAR_PLAN_SEPARATE_EC
            if plan.tile_n not in (128, 256):
                plan.tile_n, plan.tile_m = 128, 256
            spear.spear_plan_update(plan, M, N, K, r)
        ws = spear.alloc_workspace(plan.workspace_bytes)
        stream = torch.cuda.Stream()

        def call(i):
            p, s, z, A, B, wg = sets[i % 3]
            ec = spear.EC(A, B, wg, L.b_g) if use_ec else None
            spear.spear_w4ec_gemm(x, p, s, z, ec, y=y, workspace=ws, plan=plan, stream=stream)

        with torch.cuda.stream(stream):
            for i in range(3):
                call(i)
        stream.synchronize()
        n = 6
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        with torch.cuda.stream(stream):
            e0.record(stream)
            for i in range(n):
                call(i)
            e1.record(stream)
        e1.synchronize()
        t = e0.elapsed_time(e1) / 1e3 / n
        res[variant] = {"us": t * 1e6, "TFLOPs": layer_flops(M, N, K, r if use_ec else 0) / t / 1e12,
                        "plan": {"kernel": plan.kernel_id, "tile_n": plan.tile_n, "tile_m": plan.tile_m,
                                 "split_k": plan.split_k, "flags": plan.flags}}
    res["ec_overhead"] = res["ec"]["us"] / res["no_ec"]["us"] - 1.0
    res["ec_semifused_overhead"] = res["ec_semifused"]["us"] / res["no_ec"]["us"] - 1.0
    return res


def sweep_plans(args):
    """Time each valid (tile_n, split_k) decode plan in a chained CUDA graph of layer calls."""
    import torch
    import w4_gemm_error_channel_b200 as spear
    from synthetic import config_layers
    torch.cuda.set_device(0)
    if args.workload in SWEEP_ONLY:
        cfg, batches = SWEEP_ONLY[args.workload]
        shapes = config_layers(cfg, M=max(batches), layers=(0,))        # layer 0 carries an EC
    else:
        cfg, batches, kind = WORKLOADS[args.workload]
        shapes = config_layers(cfg, M=max(batches))[:1]
    if args.batches:
        batches = [int(b) for b in args.batches.split(",")]
    rows = []
    for L in shapes:
        rows += _sweep_shape(torch, spear, L, batches)
    print(json.dumps({"workload": args.workload, "sweep": rows}))


def _sweep_shape(torch, spear, L, batches):
    N, K, r = L.N, L.K, L.rank
    per_set = layer_bytes(max(batches), N, K, r)
    copies = max(2, int(np.ceil(2 * L2_BYTES / per_set)) + 1)
    sets = make_device_layer(torch, spear, L, copies)
    tiled = []

    def tiled_sets():
        # The same weight sets with the codes in tile order (made on first use).
        if not tiled and L.N % 128 == 0 and L.K % 128 == 0:
            tiled.extend((spear.spear_tile_w4(p),) + tuple(rest) for p, *rest in sets)
            torch.cuda.synchronize()
        return tiled
    dev = torch.device("cuda")
    stream = torch.cuda.Stream()
    rows = []
    for M in batches:
        x = torch.from_numpy(L.x(M).view(np.int16)).to(dev).view(torch.bfloat16)
        y = torch.empty((M, N), dtype=torch.bfloat16, device=dev)
        base = spear.spear_gemm_plan(M, N, K, r)
        # Room for the tcgen05 kernel's u buffer (bf16 [M, r]) and the fp32 main term of the
        # separate EC pass ([min(M, 256), N]) or of the semi-fused prefill path ([M, N]).
        ws = spear.alloc_workspace(base.workspace_bytes + (M * r * 2 + 255) // 256 * 256 + M * N * 4 + (8 << 20))
        # (kernel, tile_n, split_k, flags[, tile_m]): every split-K decode tiling, fused and with the
        # separate EC pass, and the tcgen05 kernel with 128- or 256-token tiles, fused and
        # semi-fused (flags 1).
        candidates = [] if M >= 1024 else [(1, tile_n, split, fl) for tile_n in (16, 32, 64, 128)
                                           for split in (1, 2, 4, 8) for fl in (0, 1)]
        for fl in ((0, 1) if M >= 128 else (0,)):
            candidates += [(2, 128, 1, fl, 128)] + ([(2, 128, 1, fl, 256)] if M >= 256 else [])
        # The tcgen05 kernel with its K range split over a cluster of 2, 4 or 8 CTAs, where its
        # grid (weight tiles x token blocks) leaves SMs idle.
        if M >= 32:
            for bn in ((128, 256) if M >= 256 else (128,)):
                grid = (N // 128) * -(-M // bn)
                candidates += [(2, 128, sk, 0, bn) for sk in (2, 4, 8) if grid * sk <= 4 * 148]
        # The register-path stream kernel (kernel 4) up to 64 tokens: token tile (8-token tiles from
        # M <= 8, 64 only with the deep ring), K codes per stage, and the ring mode (flags 2: one CTA
        # per SM with a deep ring).  The tcgen05 stream kernel (kernel 3) is slower on every measured
        # shape and is left out of the sweep.
        if M <= 64:
            bn = 16 if M <= 16 else (32 if M <= 32 else 64)
            bn_rk = 8 if M <= 8 else bn
            # (codes in the tile order of spear_tile_w4: flag 4)
            candidates += [(4, 128, kc, fl | 4, bn_rk) for kc in (128, 256) for fl in (0, 2)
                           if K % kc == 0 and (bn_rk < 64 or fl == 2) and (r <= 128)]
        for cand in candidates:
                kernel_id, tile_n, split, fl = cand[:4]
                tc_tile_m = cand[4] if len(cand) > 4 else None
                for use_ec in (True, False):
                    if (fl & spear.SPEAR_PLAN_SEPARATE_EC) and not use_ec:
                        continue
                    plan = spear.spear_plan.from_buffer_copy(base)
                    plan.kernel_id, plan.tile_n, plan.split_k, plan.flags = kernel_id, tile_n, split, fl
                    if kernel_id in (2, 3, 4):
                        plan.tile_m = tc_tile_m
                    elif base.kernel_id == 2:
                        plan.tile_m = 8 if M <= 8 else (16 if M <= 16 else 32)
                    n_calls = 64

                    src = tiled_sets() if fl & spear.SPEAR_PLAN_W4_TILES else sets

                    def call(i):
                        p, sc, z, A, B, wg = src[i % copies]
                        ec = spear.EC(A, B, wg, L.b_g) if use_ec else None
                        spear.spear_w4ec_gemm(x, p, sc, z, ec, y=y, workspace=ws, plan=plan, stream=stream)
                    try:
                        with torch.cuda.stream(stream):
                            call(0)
                        stream.synchronize()
                    except spear.SpearError:
                        continue
                    desc = (f"M={M} N={N} K={K} ec={int(use_ec)} kernel={kernel_id} tile_n={tile_n} split_k={split} "
                            f"tile_m={plan.tile_m} flags={fl}")
                    err = spear.spear_get_device_status(ws, clear=True, stream=stream)
                    if err != spear.SPEAR_OK:
                        # A bounded in-kernel wait gave up: report it and do not time this plan.
                        print(f"sweep: {desc}: device status {err}, skipped", file=sys.stderr, flush=True)
                        ws.zero_()
                        torch.cuda.synchronize()
                        continue
                    g = torch.cuda.CUDAGraph()
                    with torch.cuda.stream(stream):
                        with torch.cuda.graph(g, stream=stream):
                            for i in range(n_calls):
                                call(i)
                    best = 1e9
                    for _ in range(5):
                        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                        with torch.cuda.stream(stream):
                            e0.record(stream)
                            g.replay()
                            e1.record(stream)
                        e1.synchronize()
                        best = min(best, e0.elapsed_time(e1) * 1e3 / n_calls)
                    del g
                    print(f"sweep: {desc}: {best:.2f} us", file=sys.stderr, flush=True)
                    rows.append({"M": M, "N": N, "K": K, "rank": r if use_ec else 0, "kernel": kernel_id, "flags": fl,
                                 "tile_n": tile_n, "tile_m": plan.tile_m,
                                 "split_k": split, "us": best,
                                 "GBps": layer_bytes(M, N, K, r if use_ec else 0) / best / 1e3})
    del sets, tiled
    torch.cuda.empty_cache()
    return rows


def run_once(args):
    """Five untimed calls of one layer of the workload (the launches a profiler captures)."""
    import torch
    import w4_gemm_error_channel_b200 as spear
    from synthetic import config_layers
    torch.cuda.set_device(0)
    if args.workload in SWEEP_ONLY:
        # One linear of the 16-layer model (--linear: 0 qkv, 1 o, 2 up+gate, 3 down) of layer 0.
        cfg = SWEEP_ONLY[args.workload][0]
        M = args.once
        L = config_layers(cfg, M=M, layers=(0,))[args.linear]
    else:
        cfg, batches, kind = WORKLOADS[args.workload]
        M = args.once
        L = config_layers(cfg, M=M)[0]
    packed, scale, zero = spear.spear_pack_w4(torch.from_numpy(L.W).cuda())
    bf = lambda a: torch.from_numpy(a.view(np.int16)).cuda().view(torch.bfloat16)
    ec = None if args.no_ec else spear.EC(bf(L.A_bits), bf(L.B_bits), bf(L.wg_bits), L.b_g)
    x = bf(L.x(M))
    rank = 0 if args.no_ec else L.rank
    plan = spear.spear_gemm_plan(M, L.N, L.K, rank)
    if args.plan:
        plan.kernel_id, plan.tile_n, plan.tile_m, plan.split_k, plan.flags = (int(v) for v in args.plan.split(","))
        plan = spear.spear_plan_update(plan, M, L.N, L.K, rank)
    ws = spear.alloc_workspace(plan.workspace_bytes)
    y = torch.empty((M, L.N), dtype=torch.bfloat16, device="cuda")
    if plan.flags & spear.SPEAR_PLAN_W4_TILES:
        packed = spear.spear_tile_w4(packed)
    for _ in range(5):
        spear.spear_w4ec_gemm(x, packed, scale, zero, ec, y=y, workspace=ws, plan=plan)
    torch.cuda.synchronize()
    print(json.dumps({"once": args.workload, "M": M, "ec": not args.no_ec, "plan": repr(plan),
                      "device_status": spear.spear_get_device_status(ws)}))


def svd_demo(args):
    """Static SVD-initialised compensator (gate held at 1) on the workload's layer, M = its largest
    decode batch: the share of the 4-bit layer's output error it removes against fp64 x W^T, and
    its device time per call in a chained CUDA graph, for ranks 16..128."""
    import torch
    import w4_gemm_error_channel_b200 as spear
    from w4_gemm_error_channel_b200.svd_init import svd_compensator
    from synthetic import config_layers, f32_from_bf16_bits
    torch.cuda.set_device(0)
    cfg, batches, kind = WORKLOADS[args.workload]
    M = max(b for b in batches if b <= 64)
    L = config_layers(cfg, M=M)[0]
    dev = torch.device("cuda")
    W = torch.from_numpy(L.W).to(dev)
    packed, scale, zero = spear.spear_pack_w4(W)
    x = torch.from_numpy(L.x(M).view(np.int16)).to(dev).view(torch.bfloat16)
    xf = f32_from_bf16_bits(L.x(M)).astype(np.float64)
    y_fp = xf @ L.W.astype(np.float64).T
    stream = torch.cuda.Stream()

    def timed(ec):
        lay = spear.W4ECLayer(packed, scale, zero, ec, y_dtype=torch.float32)
        y = lay(x, stream=stream)
        stream.synchronize()
        g = torch.cuda.CUDAGraph()
        with torch.cuda.stream(stream):
            with torch.cuda.graph(g, stream=stream):
                for _ in range(32):
                    lay(x, y=y, stream=stream)
        best = 1e9
        for _ in range(5):
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            with torch.cuda.stream(stream):
                e0.record(stream)
                g.replay()
                e1.record(stream)
            e1.synchronize()
            best = min(best, e0.elapsed_time(e1) * 1e3 / 32)
        del g
        return y.double().cpu().numpy(), best

    y_w4, t_w4 = timed(None)
    rows = [{"rank": 0, "gap_recovered": 0.0, "us": t_w4}]
    for r in (16, 32, 64, 128):
        ec = svd_compensator(W, packed, scale, zero, r)
        y, t = timed(ec)
        removed = 1.0 - float(np.linalg.norm(y - y_fp) / np.linalg.norm(y_w4 - y_fp))
        rows.append({"rank": r, "gap_recovered": removed, "us": t})
    print(json.dumps({"svd_demo": {"workload": f"{args.workload}: M={M}, N={L.N}, K={L.K}, synthetic",
                                   "error": "|y - x W^T|_F relative to the plain 4-bit layer's",
                                   "ranks": rows}}))


def _sweep_model(torch, spear, Mmax):
    """The 16-layer model of config 4 on the device: (N, K, rank, W4ECLayer) per linear in model
    order (distinct W4 weights per linear, 512 MiB in all), and synthetic x per K, y per N."""
    from synthetic import make_layer
    from synthetic.workloads import SWEEP_EC_LAYERS, SWEEP_LAYERS, SWEEP_LINEARS, SWEEP_RANK
    dev = torch.device("cuda")
    bf = lambda a: torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).to(dev).view(torch.bfloat16)
    linears = []
    for layer in range(SWEEP_LAYERS):
        for li, (lname, N, K) in enumerate(SWEEP_LINEARS):
            rank = SWEEP_RANK if layer in SWEEP_EC_LAYERS else 0
            L = make_layer(f"L{layer}.{lname}", np.random.SeedSequence([1004, layer, li]), 1, N, K, rank,
                           outlier_frac=0.01, outlier_scale=20.0)
            W = torch.from_numpy(L.W).to(dev)
            packed, scale, zero = spear.spear_pack_w4(W)
            del W
            ec = spear.EC(bf(L.A_bits), bf(L.B_bits), bf(L.wg_bits), L.b_g) if rank else None
            # Both code orders at hand: the layer plans each batch size on the faster one.
            tiled = spear.spear_tile_w4(packed) if N % 128 == 0 and K % 128 == 0 else None
            linears.append((N, K, rank, spear.W4ECLayer(packed, scale, zero, ec, tiled=tiled)))
    xs = {K: bf(make_layer(f"x{K}", 1004 + K, Mmax, 128, K, 0, outlier_frac=0.01, outlier_scale=20.0).x_bits)
          for K in sorted({K for (_, K, _, _) in linears})}
    ys = {N: torch.empty((Mmax, N), dtype=torch.bfloat16, device=dev) for N in sorted({N for (N, _, _, _) in linears})}
    return linears, xs, ys


def _time_calls(torch, stream, calls, reps):
    """Device time (s) of one run of `calls` (a list of thunks), captured as one CUDA graph."""
    def run():
        for c in calls:
            c()
    with torch.cuda.stream(stream):
        run()
    stream.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.stream(stream):
        with torch.cuda.graph(g, stream=stream):
            run()
        for _ in range(2):                   # warm replays on the timed stream, finished before timing
            g.replay()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with torch.cuda.stream(stream):
        e0.record(stream)
        for _ in range(reps):
            g.replay()
        e1.record(stream)
    e1.synchronize()
    del g
    return e0.elapsed_time(e1) / 1e3 / reps


def slo_check(args):
    """The SLO-constrained chunk picker on the 16-layer model of config 4 with 16 decode tokens:
    for each ITL target, the chunk picked from a latency table, the predicted step time and the
    device time of the real step (one CUDA graph of all 64 linears on 16 + chunk tokens).  Two
    tables: the built-in one (each shape's calls measured on their own) and one measured inside
    this model (per linear type, its calls in model order on this model's weights)."""
    import torch
    import w4_gemm_error_channel_b200 as spear
    torch.cuda.set_device(0)
    D, Mmax, granule = 16, 4096, 128
    linears, xs, ys = _sweep_model(torch, spear, Mmax)
    stream = torch.cuda.Stream()
    types = {}
    for (N, K, rank, lay) in linears:
        types.setdefault((N, K, rank), []).append(lay)
    desc = [(N, K, rank, len(lays)) for (N, K, rank), lays in sorted(types.items())]

    def step_us(M):
        calls = [(lambda lay=lay, N=N, K=K: lay(xs[K][:M], y=ys[N][:M], stream=stream)) for (N, K, _, lay) in linears]
        return _time_calls(torch, stream, calls, 10 if M <= 512 else 3) * 1e6

    lut = []
    for M in (16, 144, 528, 1040, 2064, 4096):
        for (N, K, rank), lays in sorted(types.items()):
            calls = [(lambda lay=lay, N=N, K=K: lay(xs[K][:M], y=ys[N][:M], stream=stream)) for lay in lays]
            t = _time_calls(torch, stream, calls, 10 if M <= 512 else 3)
            lut.append((M, N, K, int(rank > 0), t * 1e6 / len(lays)))
    rows = []
    for table, tname in ((None, "built-in"), (lut, "in-model")):
        for slo in (1000.0, 2000.0, 4000.0, 8000.0, 12000.0):
            chunk, pred = spear.spear_pick_prefill_chunk(desc, D, Mmax - D, slo, granule=granule, lut=table)
            meas = step_us(D + chunk)
            nxt = step_us(D + chunk + granule) if D + chunk + granule <= Mmax else None
            rows.append({"table": tname, "slo_us": slo, "chunk": chunk, "predicted_us": pred, "measured_us": meas,
                         "meets_slo": meas <= slo, "next_chunk_measured_us": nxt})
    print(json.dumps({"slo_check": {"workload": "16 layers x (qkv 6144x2048, o 2048x2048, up 16384x2048, "
                                                "down 2048x8192), EC r=32 on layers 0, 1, 7, 15, 16 decode tokens, "
                                                f"chunk granule {granule}, synthetic",
                                    "in_model_table": lut, "picks": rows}}))


def kernel_name(spear, p):
    if p.kernel_id == spear.SPEAR_KERNEL_TC05:
        return "tcgen05" if p.split_k <= 1 else f"tcgen05, K split {p.split_k}"
    if p.kernel_id == spear.SPEAR_KERNEL_STREAM_RK:
        return "stream-K register path (tile order)"
    if p.kernel_id == spear.SPEAR_KERNEL_STREAM:
        return "stream-K tcgen05"
    return "split-K decode"


def launches_per_call(spear, p, M, has_ec):
    """This library's kernel launches for one spear_w4ec_gemm call with plan p."""
    sep = has_ec and p.flags & spear.SPEAR_PLAN_SEPARATE_EC
    if p.kernel_id == spear.SPEAR_KERNEL_TC05:
        return 3 if sep else 1                        # semi-fused: EC tiles, main tiles, u B add
    if p.kernel_id == spear.SPEAR_KERNEL_SPLITK:
        chunks = (M + 255) // 256                     # launches of at most 256 tokens
        return chunks * (2 if sep else 1)
    return 1                                          # the stream-K kernels


def model_pass_rows(torch, spear, batches=(1, 16, 256, 4096)):
    """Config 4: one pass over the 64 linears of the 16-layer model (qkv, o, up+gate, down per
    layer; compensators of rank 32 on layers 0, 1, 7, 15) per M, each call planned by the layer
    (spear_gemm_plan_formats over both code orders).  Weights are distinct per linear (512 MiB of
    W4 in each order, > 2x L2); each linear reads a synthetic x of its K.  Timed as a CUDA graph of
    the whole pass."""
    Mmax = max(batches)
    linears, xs, ys = _sweep_model(torch, spear, Mmax)
    peaks = json.load(open(os.path.join(ROOT, "MEASURED_PEAKS.json"))) if os.path.exists(
        os.path.join(ROOT, "MEASURED_PEAKS.json")) else {}
    hbm = peaks.get("hbm_gbs", 6650.0)
    tc = peaks.get("bf16_tflops_sustained", peaks.get("bf16_tflops", 1590.0))
    stream = torch.cuda.Stream()
    rows = []
    for M in batches:
        kinds = {}
        for (N, K, rank, lay) in linears:
            key = kernel_name(spear, lay.plan(M))
            kinds[key] = kinds.get(key, 0) + 1

        def one_pass():
            for (N, K, rank, lay) in linears:
                lay(xs[K][:M], y=ys[N][:M], stream=stream)
        with torch.cuda.stream(stream):
            one_pass()
        stream.synchronize()
        g = torch.cuda.CUDAGraph()
        with torch.cuda.stream(stream):
            with torch.cuda.graph(g, stream=stream):
                one_pass()
            for _ in range(2):               # warm replays on the timed stream, finished before timing
                g.replay()
        torch.cuda.synchronize()
        n = 10 if M <= 256 else 3
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        with torch.cuda.stream(stream):
            e0.record(stream)
            for _ in range(n):
                g.replay()
            e1.record(stream)
        e1.synchronize()
        t = e0.elapsed_time(e1) / 1e3 / n
        del g
        byts = sum(layer_bytes(M, N, K, r) for (N, K, r, _) in linears)
        flops = sum(layer_flops(M, N, K, r) for (N, K, r, _) in linears)
        bound = max(byts / (hbm * 1e9), flops / (tc * 1e12))
        status = max(spear.spear_get_device_status(lay.workspace) for (_, _, _, lay) in linears)
        rows.append({"M": M, "us_per_pass": t * 1e6, "GBps": byts / t / 1e9, "TFLOPs": flops / t / 1e12,
                     "roofline_frac": bound / t, "bound": "hbm" if byts / (hbm * 1e9) >= flops / (tc * 1e12) else "tensor",
                     "kernels": kinds, "device_status": status})
    del linears, xs, ys
    torch.cuda.empty_cache()
    return {"workload": "16 layers x (qkv 6144x2048, o 2048x2048, up 16384x2048, down 2048x8192), EC r=32 on "
                        "layers 0, 1, 7, 15, synthetic",
            "peaks": {"hbm_gbs": hbm, "bf16_tflops": tc, "note": "sustained bf16 peak"}, "passes": rows}


def model_sweep(args):
    """The 16-layer model pass for M in {1, 16, 256, 4096} (model_pass_rows), printed alone."""
    import torch
    import w4_gemm_error_channel_b200 as spear
    torch.cuda.set_device(0)
    print(json.dumps({"model_sweep": model_pass_rows(torch, spear)}))


def layer_detail(torch, spear, workload, batches):
    """Per batch size M of one workload layer: device time per call with and without the
    compensator (64 chained calls in a CUDA graph, weights rotating over copies larger than 2x
    L2), GB/s of algorithmic bytes, and the plan the layer chose over both code orders."""
    from synthetic import config_layers
    cfg = WORKLOADS[workload][0]
    L = config_layers(cfg, M=max(batches))[0]
    N, K, r = L.N, L.K, L.rank
    copies = max(2, int(np.ceil(2 * L2_BYTES / layer_bytes(max(batches), N, K, r))) + 1)
    sets = make_device_layer(torch, spear, L, copies)
    tiled = [spear.spear_tile_w4(p) for (p, *_) in sets]
    dev = torch.device("cuda")
    stream = torch.cuda.Stream()
    out = {}
    for M in batches:
        x = torch.from_numpy(L.x(M).view(np.int16)).to(dev).view(torch.bfloat16)
        y = torch.empty((M, N), dtype=torch.bfloat16, device=dev)
        row = {}
        for use_ec in (True, False):
            lays = [spear.W4ECLayer(p, sc, z, spear.EC(A, B, wg, L.b_g) if use_ec else None, tiled=t)
                    for (p, sc, z, A, B, wg), t in zip(sets, tiled)]
            plan = lays[0].plan(M)
            calls = [(lambda lay=lays[i % copies]: lay(x, y=y, stream=stream)) for i in range(64)]
            t = _time_calls(torch, stream, calls, 3) / 64
            rr = r if use_ec else 0
            key = "" if use_ec else "_no_ec"
            row["us" + key] = t * 1e6
            row["GBps" + key] = layer_bytes(M, N, K, rr) / t / 1e9
            row["plan" + key] = {"kernel": kernel_name(spear, plan), "tile_n": plan.tile_n, "tile_m": plan.tile_m,
                                 "split_k": plan.split_k, "flags": plan.flags}
            row["device_status" + key] = spear.spear_get_device_status(lays[0].workspace)
        row["ec_overhead"] = row["us"] / row["us_no_ec"] - 1.0
        out[str(M)] = row
    del sets, tiled
    torch.cuda.empty_cache()
    return {"workload": f"{workload}: N={N}, K={K}, EC rank {r}", "per_M": out}


def grouped_compare(args):
    """Device time per call of the decode-qo layer (4096 x 4096, EC r = 64) with per-channel scales
    (the dispatcher's plan) and with group-wise scales (groups of 128), EC on and off, M in
    {1, 16, 256}: a chained CUDA graph of 32 calls over rotating weight copies, best of 5."""
    import torch
    import w4_gemm_error_channel_b200 as spear
    from synthetic import config_layers
    torch.cuda.set_device(0)
    dev = torch.device("cuda")
    G = 128
    L = config_layers(1, M=256)[0]
    N, K, r = L.N, L.K, L.rank
    bf = lambda a: torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).to(dev).view(torch.bfloat16)
    W = torch.from_numpy(L.W).to(dev)
    copies = max(2, int(np.ceil(2 * L2_BYTES / layer_bytes(256, N, K, r))) + 1)
    pc = [spear.spear_pack_w4(W) for _ in range(copies)]
    gp = [spear.spear_pack_w4_grouped(W, G) for _ in range(copies)]
    del W
    A, B, wg = bf(L.A_bits), bf(L.B_bits), bf(L.wg_bits)
    stream = torch.cuda.Stream()
    rows = []
    for M in (1, 16, 256):
        x = bf(L.x(M))
        y = torch.empty((M, N), dtype=torch.bfloat16, device=dev)
        for grouped in (False, True):
            for use_ec in (True, False):
                ec = spear.EC(A, B, wg, L.b_g) if use_ec else None
                rk = r if use_ec else 0
                if grouped:
                    ws = spear.alloc_workspace(spear.spear_grouped_workspace_bytes(M, N, K, G, rk))
                    call = lambda i: spear.spear_w4ec_gemm_grouped(x, *gp[i % copies], G, ec, y=y, workspace=ws,
                                                                   stream=stream)
                else:
                    plan = spear.spear_gemm_plan(M, N, K, rk)
                    ws = spear.alloc_workspace(plan.workspace_bytes)
                    call = lambda i: spear.spear_w4ec_gemm(x, *pc[i % copies], ec, y=y, workspace=ws, plan=plan,
                                                           stream=stream)
                n = 32
                with torch.cuda.stream(stream):
                    call(0)
                stream.synchronize()
                g = torch.cuda.CUDAGraph()
                with torch.cuda.stream(stream):
                    with torch.cuda.graph(g, stream=stream):
                        for i in range(n):
                            call(i)
                best = 1e9
                for _ in range(5):
                    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                    with torch.cuda.stream(stream):
                        e0.record(stream)
                        g.replay()
                        e1.record(stream)
                    e1.synchronize()
                    best = min(best, e0.elapsed_time(e1) * 1e3 / n)
                del g
                extra = (N * (K // G) * 4 - 4 * N) if grouped else 0          # group scales and zeros
                byts = layer_bytes(M, N, K, rk) + extra
                rows.append({"M": M, "scales": f"group {G}" if grouped else "per channel", "ec": use_ec,
                             "us": best, "GBps": byts / best / 1e3,
                             "device_status": spear.spear_get_device_status(ws)})
    print(json.dumps({"grouped_compare": {"workload": f"decode-qo layer {N}x{K}, EC r={r}, synthetic", "rows": rows}}))


def gate_compare(args):
    """Device time per call of the same layer with the scalar gate and with the bottleneck-MLP gate
    (H = 16, random fp32 gate weights), in a chained CUDA graph of calls over rotating weight copies."""
    import torch
    import w4_gemm_error_channel_b200 as spear
    from synthetic import config_layers
    torch.cuda.set_device(0)
    dev = torch.device("cuda")
    stream = torch.cuda.Stream()
    rows = []
    for wname, M in (("decode-qo", 16), ("prefill", 2048)):
        cfg = WORKLOADS[wname][0]
        L = config_layers(cfg, M=M)[0]
        per_set = layer_bytes(M, L.N, L.K, L.rank)
        copies = max(2, int(np.ceil(2 * L2_BYTES / per_set)) + 1)
        sets = make_device_layer(torch, spear, L, copies)
        x = torch.from_numpy(L.x(M).view(np.int16)).to(dev).view(torch.bfloat16)
        y = torch.empty((M, L.N), dtype=torch.bfloat16, device=dev)
        rng = np.random.default_rng(5)
        H = 16
        gate = [torch.from_numpy((rng.standard_normal(sh) * 0.3).astype(np.float32)).to(dev)
                for sh in ((H, L.rank), (H,), (L.rank, H), (L.rank,))]
        res = {"workload": f"{wname} M={M}", "rank": L.rank, "hidden": H}
        for kind in ("scalar", "mlp"):
            def ec_of(A, B, wg):
                if kind == "scalar":
                    return spear.EC(A, B, wg, L.b_g)
                return spear.EC(A, B, wg, L.b_g, gate_w1=gate[0], gate_b1=gate[1], gate_w2=gate[2],
                                gate_b2=gate[3], alpha=1.0)
            layers = [spear.W4ECLayer(p, s_, z, ec_of(A, B, wg)) for (p, s_, z, A, B, wg) in sets]
            n = 32 if M <= 64 else 8
            with torch.cuda.stream(stream):
                for lay in layers:
                    lay(x, y=y, stream=stream)
            stream.synchronize()
            g = torch.cuda.CUDAGraph()
            with torch.cuda.stream(stream):
                with torch.cuda.graph(g, stream=stream):
                    for i in range(n):
                        layers[i % copies](x, y=y, stream=stream)
            best = 1e9
            for _ in range(5):
                e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                with torch.cuda.stream(stream):
                    e0.record(stream)
                    g.replay()
                    e1.record(stream)
                e1.synchronize()
                best = min(best, e0.elapsed_time(e1) * 1e3 / n)
            del g
            res[f"us_{kind}"] = best
            res[f"status_{kind}"] = max(spear.spear_get_device_status(lay.workspace) for lay in layers)
        rows.append(res)
        del sets
        torch.cuda.empty_cache()
    print(json.dumps({"gate_compare": rows}))


def main():
    args = parse()
    if args.gate_compare:
        gate_compare(args)
        return
    if args.grouped_compare:
        grouped_compare(args)
        return
    if args.model_sweep:
        model_sweep(args)
        return
    if args.svd_demo:
        svd_demo(args)
        return
    if args.once:
        run_once(args)
        return
    if args.slo_check:
        slo_check(args)
        return
    if args.sweep:
        sweep_plans(args)
        return
    if args.workload in SWEEP_ONLY:
        raise SystemExit(f"--workload {args.workload} is for --sweep only")
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    cfg, batches, kind = WORKLOADS[args.workload]

    if args.impl == "reference":
        # The reference arm is the CPU oracle (the pages ship no implementation).  Rank 0 only.
        if rank != 0:
            return
        r = oracle_sample(args.workload, min(args.cpu_seconds, 15.0) / max(1, args.steps) * args.steps, batches)
        if kind == "prefill":
            val, unit = r["flops"] / r["seconds"] / 1e12, "TFLOP/s"
        else:
            val, unit = r["bytes"] / r["seconds"] / 1e9, "GB/s"
        from synthetic import config_layers
        L = config_layers(cfg, M=1)[0]
        out = {"impl": "reference",
               "metric": "W4+gated-EC GEMM: decode GB/s and prefill TFLOP/s vs B200 roofline, 1 GPU",
               "value": val, "unit": unit, "n_gpus": 1, "steps": args.steps, "warmup": args.warmup,
               "ms_per_step": r["seconds"] / r["reps"] * 1e3, "higher_is_better": True, "scaling": "weak",
               "vs_baseline": None, "dtype": "f64", "data": "synthetic",
               "config": {"workload": f"{args.workload}: M in {batches}, N={L.N}, K={L.K}, EC rank {L.rank}"},
               "cpu_baseline": {"value": val, "unit": unit, "cores": r["cores"], "kind": "oracle",
                                "sample": f"{r['reps']} passes over M={r['M']}, {r['seconds']:.1f} s"},
               "e2e": {"value": val, "unit": unit, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
        print(json.dumps(out))
        return

    # Build the CPU baseline before any CUDA work (the oracle uses OpenMP threads).
    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = cpu_baseline_obj(args.workload, args.cpu_seconds)

    import torch
    dist = None
    if world > 1:
        import datetime
        import torch.distributed as dist
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    else:
        torch.cuda.set_device(0)
    out = run_ours(args, rank, world, torch, dist)
    if world == 1 and args.workload == "decode-qo" and not args.no_detail:
        # Secondary per-shape figures (one GPU only): the decode-mlp layer at M in {1, 8, 32, 64}
        # and one pass of the 16-layer model at M in {1, 16, 256, 4096}.
        import w4_gemm_error_channel_b200 as spear
        try:
            out["detail_decode_mlp"] = layer_detail(torch, spear, "decode-mlp", [1, 8, 32, 64])
        except Exception as e:
            out["detail_decode_mlp"] = {"error": str(e)}
        try:
            out["detail_model_pass"] = model_pass_rows(torch, spear)
        except Exception as e:
            out["detail_model_pass"] = {"error": str(e)}
    if rank == 0 and not args.no_prefill and args.workload != "prefill":
        import w4_gemm_error_channel_b200 as spear
        try:
            out["prefill"] = prefill_summary(torch, spear)
        except Exception as e:  # secondary figure only; the main line stands on its own
            out["prefill"] = {"error": str(e)}
    if cpu is not None:
        out["cpu_baseline"] = cpu
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    if rank == 0:
        print(json.dumps(out))


if __name__ == "__main__":
    main()
