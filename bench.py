#!/usr/bin/env python3
"""Benchmark of the sm_100a fused attention forward pass.

One step = one forward pass of the workload in BOTH masking modes (the
non-causal and the causal call, inputs resident in HBM).  Rank 0 prints one
JSON line:

  value        whole-job TFLOP/s (4*B*H*N^2*d non-causal + 2*B*H*N^2*d causal per
               step, summed over ranks, divided by the max over ranks of the
               device-timed region)
  e2e          the same metric through the host-buffer entry point (pinned host
               Q/K/V copied in, O/LSE copied out, inside the timed region)
  roofline     the attention kernel against the measured dense bf16 peak
  cpu_baseline the fp64 oracle on the host cores, on a bounded sample of rows

`--impl reference` times the fp64 oracle instead (the reference arm of this
build: there is no other implementation of the pages to run).

Multi-GPU (`torchrun --nproc-per-node N bench.py --gpus N`): the work is
independent (batch, head) slices, so every rank runs its own replica of the
workload with no data-path collective (weak scaling).
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import re
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "attention fwd TFLOP/s (causal/non-causal) and % of B200 dense BF16 peak"
DATASHEET_BF16_TFLOPS = 2250.0

WORKLOADS = {
    # the headline workload: N >= 4096, d = 128, both masking modes, wide score range
    "b1_h32_n16384_d128_qk_sigma3": dict(B=1, H=32, N=16384, d=128, sigma_qk=3.0),
    # the same shape with unit-variance scores (the rescale-cost A/B against the line above)
    "b1_h32_n16384_d128": dict(B=1, H=32, N=16384, d=128, sigma_qk=1.0),
    "b2_h16_n4096_d128": dict(B=2, H=16, N=4096, d=128, sigma_qk=1.0),
    "b1_h32_n16384_d64": dict(B=1, H=32, N=16384, d=64, sigma_qk=1.0),
    "b4_h16_n4096_d64": dict(B=4, H=16, N=4096, d=64, sigma_qk=1.0),
    "b4_h8_n1024_d64": dict(B=4, H=8, N=1024, d=64, sigma_qk=1.0),
    # profiling size: Q, K, V, O = 4 x 64 MiB, above the L2, a short launch
    "b1_h64_n4096_d128": dict(B=1, H=64, N=4096, d=128, sigma_qk=1.0),
}
MODES = {"both": (False, True), "non-causal": (False,), "causal": (True,)}
DEFAULT_WORKLOAD = "b1_h32_n16384_d128_qk_sigma3"


def flops(B, H, N, d, causal):
    f = 4.0 * B * H * N * N * d
    return f / 2 if causal else f


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            p = json.load(f)
        return dict(bf16=float(p["bf16_tflops"]), bf16_sustained=float(p["bf16_tflops_sustained"]),
                    hbm=float(p["hbm_gbs"]), source="measured")
    except Exception:
        return dict(bf16=1590.0, bf16_sustained=1400.0, hbm=6650.0, source="fallback")


KERNEL_FAMILY = {0: "fa_fwd_kernel", 1: "fa_fwd_pp_kernel", **{a: "fa_fwd_2q_kernel" for a in range(2, 18)}}


def measured_traffic(workload, algorithm=0):
    """DRAM bytes per non-causal launch from the committed ncu summary of the
    kernel family the headline runs (algorithm 0: fa_fwd_kernel, 1: the split-KV
    ping-pong kernel, 2-5: the two-query-tile kernel), or None when that kernel's
    source changed since the counters were taken (or the summary does not cover
    this workload)."""
    if workload != DEFAULT_WORKLOAD:
        return None, None
    name = KERNEL_FAMILY[algorithm]
    prof = os.path.join(ROOT, "profiles", f"{name}_b1_h64_n4096_d128_ncu.md")
    src = os.path.join(ROOT, "attention_forward_17_b200", "csrc", f"{name}.cuh")
    try:
        text = open(prof).read()
        want = re.search(r"kernel_source_sha256_16: (\w+)", text).group(1)
        have = hashlib.sha256(open(src, "rb").read()).hexdigest()[:16]
        if want != have:
            return None, "kernel changed since the ncu capture"
        val = float(re.search(r"traffic_bytes_per_launch_noncausal: ([0-9.e+]+)", text).group(1))
        return val, (f"ncu dram__bytes_read+write of one launch at B=1,H=64,N=4096,d=128, scaled x2 by "
                     f"BH*N*d to the workload (profiles/{name}_b1_h64_n4096_d128_ncu.md)")
    except (OSError, AttributeError, ValueError):
        return None, None


def profile_traffic(profile, source):
    """DRAM bytes per launch from a committed ncu summary under profiles/, or
    None when the kernel source changed since the capture."""
    try:
        text = open(os.path.join(ROOT, "profiles", profile)).read()
        want = re.search(r"kernel_source_sha256_16: (\w+)", text).group(1)
        have = hashlib.sha256(open(os.path.join(ROOT, source), "rb").read()).hexdigest()[:16]
        if want != have:
            return None
        return float(re.search(r"traffic_bytes_per_launch: ([0-9.e+]+)", text).group(1))
    except (OSError, AttributeError, ValueError):
        return None


# ------------------------------------------------------------------ clocks
def _load_clocks():
    """The package's clock sampler, loaded from its file so that the reference
    (oracle) arm does not load the CUDA library with the package."""
    import importlib.util
    spec = importlib.util.spec_from_file_location(
        "fa_b200_clocks", os.path.join(ROOT, "attention_forward_17_b200", "clocks.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


ClockSampler = _load_clocks().ClockSampler


# ------------------------------------------------------------------ CPU oracle sample
def oracle_sample(bits, cfg, target_s, seed=0):
    """Time the fp64 oracle on a bounded sample of rows of the workload, both
    modes; returns (TFLOP/s by the metric's per-row FLOP convention, details)."""
    import numpy as np
    import oracle
    q, k, v = bits
    B, H, N, d = q.shape
    scale = 1.0 / math.sqrt(d)
    rng = np.random.default_rng(seed)
    threads = oracle.default_threads()
    nrows, spent, done_flops, results = 8, 0.0, 0.0, []
    while True:
        rows = np.sort(rng.choice(B * H * N, nrows, replace=False)).astype(np.int64)
        step_flops, t0 = 0.0, time.perf_counter()
        outs = {}
        for causal in (False, True):
            outs[causal] = oracle.attention_rows(q, k, v, causal, scale, rows)
            # per-row share of the metric's FLOP convention
            step_flops += nrows * (4.0 * N * d / (2 if causal else 1))
        dt = time.perf_counter() - t0
        spent += dt
        done_flops += step_flops
        results.append((rows, outs))
        if spent >= target_s or nrows >= B * H * N // 4:
            break
        nrows = min(B * H * N // 4, max(nrows * 2, int(nrows * target_s / max(dt, 1e-3) * 0.5)))
    return done_flops / spent / 1e12, dict(seconds=spent, cores=threads, results=results,
                                           rows=sum(len(r[0]) for r in results))


def sample_parity(results, o_by_mode, lse_by_mode, d):
    """The GPU output on the oracle's sampled rows: O max-abs, O relative L2
    over the sampled rows (per mode, the worst reported) and LSE max-abs,
    against the tolerances (2e-2, 1e-2, 1e-3)."""
    import numpy as np
    worst = dict(o_max_abs=0.0, o_rel_l2=0.0, lse_max_abs=0.0)
    err2 = {}
    ref2 = {}
    for rows, outs in results:
        for causal, (o_ref, lse_ref) in outs.items():
            o = o_by_mode[causal].view(-1, d)[rows].float().cpu().numpy().astype(np.float64)
            lse = lse_by_mode[causal].view(-1)[rows].cpu().numpy().astype(np.float64)
            worst["o_max_abs"] = max(worst["o_max_abs"], float(np.abs(o - o_ref).max()))
            worst["lse_max_abs"] = max(worst["lse_max_abs"], float(np.abs(lse - lse_ref).max()))
            err2[causal] = err2.get(causal, 0.0) + float(np.sum((o - o_ref) ** 2))
            ref2[causal] = ref2.get(causal, 0.0) + float(np.sum(o_ref ** 2))
    for c in err2:
        worst["o_rel_l2"] = max(worst["o_rel_l2"], math.sqrt(err2[c] / ref2[c]) if ref2[c] > 0 else 0.0)
    worst["pass"] = (worst["o_max_abs"] <= 2e-2 and worst["o_rel_l2"] <= 1e-2
                     and worst["lse_max_abs"] <= 1e-3)
    return worst


# ------------------------------------------------------------------ arms
def dist_setup(n_gpus):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world != n_gpus:
        raise SystemExit(f"--gpus {n_gpus} but WORLD_SIZE={world}")
    return world, rank, local


def max_over_ranks(x, world, device=None):
    """Largest value of x over all ranks (the job's time is its slowest rank's)."""
    if world == 1:
        return x
    import torch
    import torch.distributed as dist
    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def run_reference(args, cfg):
    """The oracle arm: fp64 CPU attention on bounded row samples per step."""
    world, rank, _ = dist_setup(args.gpus)
    if rank != 0:
        return
    import numpy as np
    import oracle
    import seeded_inputs as si
    B, H, N, d = cfg["B"], cfg["H"], cfg["N"], cfg["d"]
    bits = si.make_qkv(B, H, N, d, seed=0, sigma_qk=cfg["sigma_qk"])
    q, k, v = bits
    scale = 1.0 / math.sqrt(d)
    rows_per_step = max(8, args.ref_rows)
    rng = np.random.default_rng(0)

    def step():
        rows = np.sort(rng.choice(B * H * N, rows_per_step, replace=False)).astype(np.int64)
        f = 0.0
        for causal in (False, True):
            oracle.attention_rows(q, k, v, causal, scale, rows)
            f += rows_per_step * 4.0 * N * d / (2 if causal else 1)
        return f

    for _ in range(args.warmup):
        step()
    t0 = time.perf_counter()
    total = sum(step() for _ in range(args.steps))
    dt = time.perf_counter() - t0
    value = total / dt / 1e12
    sample = (f"{rows_per_step} random query rows per step, each in both masking modes, of "
              f"B={B},H={H},N={N},d={d}; complete fp64 score rows")
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "TFLOP/s",
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": dt / args.steps * 1e3, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": workload_config(args.workload, cfg, args.gpus),
        "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": oracle.default_threads(),
                         "kind": "oracle", "sample": sample},
        "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def schedule_of(N, d, causal, schedule=None, causal_group=None):
    """The kernel schedule used for this problem: the search table's, unless pinned."""
    import attention_forward_17_b200 as fa
    sid, grp = fa.pick_schedule(N, d, causal)
    sid = sid if schedule is None else schedule
    grp = grp if causal_group is None else causal_group
    s = fa.schedules()[sid]
    return {"id": sid, "exp_poly_every": s["emu_every"], "kv_slots": s["kv_slots"],
            "persistent": s["persistent"], "algorithm": s["algorithm"], "key_tile": s["key_tile"],
            "causal_group": grp if (causal and s["persistent"] != 1) else None}


def workload_config(name, cfg, n_gpus, modes=(False, True)):
    return {"workload": name, "B": cfg["B"], "H": cfg["H"], "N": cfg["N"], "d": cfg["d"],
            "qk_sigma": cfg["sigma_qk"], "v_sigma": 1.0, "scale": "1/sqrt(d)",
            "modes": ["causal" if c else "non-causal" for c in modes], "seed": 0,
            "l2": "inputs (Q,K,V = 3 x {:.0f} MiB) larger than the 126 MB L2".format(
                cfg["B"] * cfg["H"] * cfg["N"] * cfg["d"] * 2 / 2 ** 20),
            "parallelism": f"replicas x{n_gpus} (independent (b,h) slices, no collective)"}


def run_ours(args, cfg):
    import torch
    world, rank, local = dist_setup(args.gpus)
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300),
                                device_id=dev)
    import numpy as np
    import attention_forward_17_b200 as fa
    # --schedule / --causal-group pin the kernel schedule (profiling); default: the search table
    override = {k: v for k, v in (("schedule", args.schedule), ("causal_group", args.causal_group))
                if v is not None}
    import seeded_inputs as si

    B, H, N, d = cfg["B"], cfg["H"], cfg["N"], cfg["d"]
    modes = MODES[args.modes]
    bits = si.make_qkv(B, H, N, d, seed=rank, sigma_qk=cfg["sigma_qk"])

    def dev_tensor(b):
        return torch.from_numpy(b.view(np.int16)).view(torch.bfloat16).to(dev)

    q, k, v = (dev_tensor(b) for b in bits)
    o = {c: torch.empty_like(q) for c in modes}
    lse = {c: torch.empty((B, H, N), dtype=torch.float32, device=dev) for c in modes}
    stream = torch.cuda.current_stream(dev)
    f_step = sum(flops(B, H, N, d, c) for c in modes)

    def barrier():
        if world > 1:
            import torch.distributed as dist
            dist.barrier()


    # ---------------- device-resident timing, per-launch events
    for _ in range(args.warmup):
        for c in modes:
            fa.fa_fwd(q, k, v, causal=c, out=o[c], lse=lse[c], **override)
    torch.cuda.synchronize()
    ev = {c: [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
              for _ in range(args.steps)] for c in modes}
    t_start, t_end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    gpu_index = local
    with ClockSampler(gpu_index) as clk:
        barrier()
        torch.cuda.synchronize()
        t_start.record(stream)
        for s in range(args.steps):
            for c in modes:
                ev[c][s][0].record(stream)
                fa.fa_fwd(q, k, v, causal=c, out=o[c], lse=lse[c], **override)
                ev[c][s][1].record(stream)
        t_end.record(stream)
        torch.cuda.synchronize()
        barrier()
    elapsed_ms = max_over_ranks(t_start.elapsed_time(t_end), world, dev)
    per_launch = {c: [a.elapsed_time(b) for a, b in ev[c]] for c in modes}
    launch_ms = {c: statistics.mean(per_launch[c]) for c in modes}
    clocks = clk.summary()
    value = world * f_step * args.steps / (elapsed_ms / 1e3) / 1e12

    # ---------------- end to end through the host-buffer entry point
    e2e = None
    if not args.no_e2e:
        host = [torch.from_numpy(b.view(np.int16)).view(torch.bfloat16).pin_memory() for b in bits]
        o_h = {c: torch.empty_like(host[0]).pin_memory() for c in modes}
        l_h = {c: torch.empty((B, H, N), dtype=torch.float32).pin_memory() for c in modes}
        qd, kd, vd = (torch.empty_like(q) for _ in range(3))
        e2e_steps = max(1, min(args.steps, 10))

        def e2e_step():
            for c in modes:
                fa.fa_fwd_host(host[0], host[1], host[2], o_h[c], l_h[c], qd, kd, vd, o[c], lse[c],
                               causal=c)

        for _ in range(max(1, min(args.warmup, 3))):
            e2e_step()
        torch.cuda.synchronize()
        barrier()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        for _ in range(e2e_steps):
            e2e_step()
        b.record(stream)
        torch.cuda.synchronize()
        barrier()
        e2e_ms = max_over_ranks(a.elapsed_time(b), world, dev)
        tensor_bytes = B * H * N * d * 2
        e2e = {"value": world * f_step * e2e_steps / (e2e_ms / 1e3) / 1e12, "unit": "TFLOP/s",
               "h2d_bytes_per_step": 2 * 3 * tensor_bytes,
               "d2h_bytes_per_step": 2 * (tensor_bytes + B * H * N * 4),
               "steps": e2e_steps, "entry_point": "fa_fwd_host"}

    # ---------------- roofline of the dominant launch (non-causal instantiation)
    peaks = load_peaks()
    ach = {c: flops(B, H, N, d, c) / (launch_ms[c] / 1e3) / 1e12 for c in modes}
    dominant = max(modes, key=lambda c: launch_ms[c])
    sch_dom = schedule_of(N, d, dominant, args.schedule, args.causal_group)
    traffic, traffic_src = measured_traffic(args.workload, sch_dom["algorithm"])
    kname = KERNEL_FAMILY[sch_dom["algorithm"]]
    roofline = {"bound": "tensor", "kernel": f"{kname} d={d} {'causal' if dominant else 'non-causal'} "
                                             f"schedule {sch_dom['id']}",
                "achieved": ach[dominant], "peak": peaks["bf16"], "unit": "TFLOP/s",
                "frac": ach[dominant] / peaks["bf16"], "peak_source": peaks["source"] + " burst",
                "traffic": traffic if dominant is False else None, "traffic_source": traffic_src,
                "algorithmic_bytes_per_launch": 8.0 * B * H * N * d + 4.0 * B * H * N,
                "per_mode": {("causal" if c else "non_causal"): {
                    "ms_per_launch": launch_ms[c], "tflops": ach[c],
                    "ms_median": statistics.median(per_launch[c]), "ms_min": min(per_launch[c]),
                    "frac_of_measured_burst": ach[c] / peaks["bf16"],
                    "frac_of_measured_sustained": ach[c] / peaks["bf16_sustained"],
                    "frac_of_datasheet_2250": ach[c] / DATASHEET_BF16_TFLOPS} for c in modes}}

    # ---------------- context: PyTorch scaled-dot-product attention on the same GPU and inputs
    # (the pages' comparator; library code, timed outside the measured region, never used for parity)
    context = None
    if not args.no_context:
        import torch.nn.functional as F
        context = {"torch_sdpa_tflops": {}, "note": "torch.nn.functional.scaled_dot_product_attention, "
                   "bf16, default backend selection, same Q/K/V, 10 launches after 3 warm-ups"}
        for c in modes:
            try:
                run = lambda: F.scaled_dot_product_attention(q, k, v, is_causal=c, scale=1.0 / math.sqrt(d))
                for _ in range(3):
                    run()
                a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                torch.cuda.synchronize()
                a.record(stream)
                for _ in range(10):
                    run()
                b.record(stream)
                torch.cuda.synchronize()
                context["torch_sdpa_tflops"]["causal" if c else "non_causal"] = \
                    flops(B, H, N, d, c) / (a.elapsed_time(b) / 10 / 1e3) / 1e12
            except Exception as exc:          # a backend may refuse a shape; context only
                context["torch_sdpa_tflops"]["causal" if c else "non_causal"] = f"unavailable: {exc}"[:120]

    # ---------------- CPU baseline (rank 0, N=1 only)
    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline and args.modes == "both":
        v_cpu, det = oracle_sample(bits, cfg, args.cpu_seconds)
        par = sample_parity(det["results"], o, lse, d)
        cpu = {"value": v_cpu, "unit": "TFLOP/s", "cores": det["cores"], "kind": "oracle",
               "sample": f"{det['rows']} random query rows of the workload, each in both masking "
                         f"modes (complete fp64 score rows), {det['seconds']:.1f} s",
               "sample_parity_vs_gpu": par}

    if rank == 0:
        line = {
            "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": elapsed_ms / args.steps,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
            "data": "synthetic",
            "config": dict(workload_config(args.workload, cfg, world, modes),
                           schedule={("causal" if c else "non-causal"):
                                     schedule_of(N, d, c, args.schedule, args.causal_group)
                                     for c in modes}),
            "pct_of_peak": {"measured_burst": 100 * value / world / peaks["bf16"],
                            "measured_sustained": 100 * value / world / peaks["bf16_sustained"],
                            "datasheet_2250": 100 * value / world / DATASHEET_BF16_TFLOPS},
            "roofline": roofline, "cpu_baseline": cpu, "e2e": e2e, "context": context,
            "gpu_launches": args.steps * len(modes) * fa.launches_per_call(B, H, N, d),
            "clocks": clocks, "impl": "ours",
        }
        print(json.dumps(line), flush=True)
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()


def bench_row_softmax(args):
    """One JSON line for the row-wise softmax kernel (HBM-bound)."""
    import numpy as np
    import torch
    import attention_forward_17_b200 as fa
    import seeded_inputs as si
    rows, cols = 32768, 4096
    bits = si.normal_bf16((rows, cols), seed=0, tensor_id=7, sigma=2.0)
    x = torch.from_numpy(bits.view(np.int16)).view(torch.bfloat16).cuda()
    y = torch.empty_like(x)
    for _ in range(args.warmup):
        fa.row_softmax(x, 1.0, out=y)
    torch.cuda.synchronize()
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    # inputs + outputs (512 MiB) exceed L2, so consecutive launches re-read HBM
    with ClockSampler(0) as clk:
        a.record()
        for _ in range(args.steps):
            fa.row_softmax(x, 1.0, out=y)
        b.record()
        torch.cuda.synchronize()
    ms = a.elapsed_time(b) / args.steps
    nbytes = 2.0 * 2 * rows * cols
    gbs = nbytes / (ms / 1e3) / 1e9
    peaks = load_peaks()
    # CPU baseline: the oracle on a sample of rows
    import oracle
    t0 = time.perf_counter()
    sample = 512
    ref = oracle.row_softmax(bits[:sample], 1.0)
    dt = time.perf_counter() - t0
    got = y[:sample].float().cpu().numpy().astype(np.float64)
    worst = float(np.max(np.abs(got - ref) / (np.abs(ref) + 1e-30)))
    line = {"metric": "row softmax GB/s (bf16 in, bf16 out)", "value": gbs, "unit": "GB/s",
            "n_gpus": 1, "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
            "data": "synthetic", "config": {"workload": f"row_softmax_r{rows}_c{cols}", "rows": rows,
                                            "cols": cols, "l2": "512 MiB moved per launch, above L2"},
            "roofline": {"bound": "hbm", "achieved": gbs, "peak": peaks["hbm"], "unit": "GB/s",
                         "frac": gbs / peaks["hbm"],
                         "traffic": profile_traffic("row_softmax_fast_r32768_c4096_ncu.md",
                                                    "attention_forward_17_b200/csrc/row_softmax.cu"),
                         "algorithmic_bytes_per_launch": nbytes},
            "cpu_baseline": {"value": sample * cols * 4 / dt / 1e9, "unit": "GB/s",
                             "cores": oracle.default_threads(), "kind": "oracle",
                             "sample": f"{sample} rows", "max_rel_err_vs_gpu": worst},
            "gpu_launches": args.steps * fa.lib.fa_row_softmax_launches(rows, cols),
            "clocks": clk.summary(), "impl": "ours"}
    print(json.dumps(line), flush=True)


def _event_loop(fn, steps):
    """Mean device time (ms) of `fn` over `steps` back-to-back launches, CUDA
    events on the current stream, with clocks sampled meanwhile."""
    import torch
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize()
    with ClockSampler(0) as clk:
        a.record()
        for _ in range(steps):
            fn()
        b.record()
        torch.cuda.synchronize()
    return a.elapsed_time(b) / steps, clk.summary()


def bench_gemm(args):
    """One JSON line for the tcgen05 GEMM with the fused bias + GELU epilogue
    (tensor-bound), with cuBLAS (torch eager) timed beside it for context."""
    import numpy as np
    import torch
    import attention_forward_17_b200 as fa
    import seeded_inputs as si
    M = N = K = 8192
    a_b, b_b, bias_b = si.make_gemm(M, N, K, seed=0)
    dev = lambda x: torch.from_numpy(np.ascontiguousarray(x).view(np.int16)).view(torch.bfloat16).cuda()
    a, b, bias = dev(a_b), dev(b_b), dev(bias_b)
    c = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
    run = lambda: fa.gemm(a, b, bias, fa.FA_GEMM_BIAS_GELU, out=c)
    for _ in range(args.warmup):
        run()
    ms, clocks = _event_loop(run, args.steps)
    flop = 2.0 * M * N * K
    tf = flop / (ms / 1e3) / 1e12
    # context: cuBLAS through torch, plain product and the eager three-kernel epilogue
    eager = lambda: torch.nn.functional.gelu(a @ b + bias)
    plain = lambda: a @ b
    for _ in range(args.warmup):
        eager(); plain()
    ms_eager, _ = _event_loop(eager, args.steps)
    ms_plain, _ = _event_loop(plain, args.steps)
    peaks = load_peaks()
    import oracle
    # CPU baseline: the oracle on sampled entries, sized to a few seconds
    rng = np.random.default_rng(0)
    n = 512
    while True:
        idx = rng.integers(0, M * N, n)
        t0 = time.perf_counter()
        ref = oracle.gemm_entries(a_b, b_b, bias_b, idx, 2)
        dt = time.perf_counter() - t0
        if dt > 2.0 or n >= 1 << 20:
            break
        n *= 4
    got = c.float().cpu().numpy().reshape(-1)[idx].astype(np.float64)
    worst = float(np.max(np.abs(got - ref) - 2.0 ** -8 * np.abs(ref)))
    line = {"metric": "GEMM + bias + GELU TFLOP/s (bf16 in, fp32 accumulate, bf16 out)",
            "value": tf, "unit": "TFLOP/s", "n_gpus": 1, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
            "config": {"workload": f"gemm_bias_gelu_m{M}_n{N}_k{K}", "M": M, "N": N, "K": K,
                       "l2": "A, B, C = 384 MiB, above L2"},
            "roofline": {"bound": "tensor", "achieved": tf, "peak": peaks["bf16"],
                         "unit": "TFLOP/s", "frac": tf / peaks["bf16"],
                         "traffic": profile_traffic("gemm2_kernel_m8192_n8192_k8192_ncu.md",
                                                    "attention_forward_17_b200/csrc/gemm_bias_gelu.cu"),
                         "algorithmic_flops_per_launch": flop,
                         "peak_source": peaks["source"] + " bf16 burst (cuBLAS 8192^3)"},
            "context": {"cublas_plain_tflops": flop / (ms_plain / 1e3) / 1e12,
                        "torch_eager_gelu_bias_tflops": flop / (ms_eager / 1e3) / 1e12},
            "cpu_baseline": {"value": len(idx) * 2.0 * K / dt / 1e12, "unit": "TFLOP/s",
                             "cores": oracle.default_threads(), "kind": "oracle",
                             "sample": f"{len(idx)} random entries of C",
                             "max_excess_err_vs_gpu": worst},
            "gpu_launches": args.steps * fa.lib.fa_gemm_launches(M, N, K),
            "clocks": clocks, "impl": "ours"}
    print(json.dumps(line), flush=True)


def bench_vector_add(args):
    """One JSON line for the fp32 vector add (HBM-bound)."""
    import numpy as np
    import torch
    import attention_forward_17_b200 as fa
    import seeded_inputs as si
    n = 1 << 28
    xh, yh = si.make_add(n, seed=0)
    x, y = torch.from_numpy(xh).cuda(), torch.from_numpy(yh).cuda()
    z = torch.empty_like(x)
    run = lambda: fa.vector_add(x, y, out=z)
    for _ in range(args.warmup):
        run()
    ms, clocks = _event_loop(run, args.steps)
    nbytes = 12.0 * n
    gbs = nbytes / (ms / 1e3) / 1e9
    peaks = load_peaks()
    import oracle
    m = 1 << 26
    t0 = time.perf_counter()
    ref = oracle.vector_add(xh[:m], yh[:m])
    dt = time.perf_counter() - t0
    exact = bool(np.array_equal(z[:m].cpu().numpy(), ref.astype(np.float32)))
    line = {"metric": "vector add GB/s (fp32)", "value": gbs, "unit": "GB/s", "n_gpus": 1,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f32",
            "data": "synthetic", "config": {"workload": f"vector_add_n{n}", "n": n,
                                            "l2": "3 GiB moved per launch, above L2"},
            "roofline": {"bound": "hbm", "achieved": gbs, "peak": peaks["hbm"], "unit": "GB/s",
                         "frac": gbs / peaks["hbm"],
                         "traffic": profile_traffic("vector_add_v4_n268435456_ncu.md",
                                                    "attention_forward_17_b200/csrc/vector_add.cu"),
                         "algorithmic_bytes_per_launch": nbytes},
            "cpu_baseline": {"value": m * 12.0 / dt / 1e9, "unit": "GB/s",
                             "cores": oracle.default_threads(), "kind": "oracle",
                             "sample": f"first {m} elements", "bit_exact_vs_gpu": exact},
            "gpu_launches": args.steps * fa.lib.fa_vector_add_launches(n),
            "clocks": clocks, "impl": "ours"}
    print(json.dumps(line), flush=True)


def bench_sweep(args):
    """Sequence-length sweep: N in 512..32768 with B = max(1, 16384/N), H = 16,
    d in {64, 128}, bf16 N(0,1), both masks; one JSON line per point with the
    TFLOP/s of each mask (mean of `--steps` launches after `--warmup`, short
    back-to-back bursts) and the fraction of the measured bf16 burst peak."""
    import numpy as np
    import torch
    import attention_forward_17_b200 as fa
    import seeded_inputs as si
    peaks = load_peaks()
    for d in (64, 128):
        for N in (512, 1024, 2048, 4096, 8192, 16384, 32768):
            B, H = max(1, 16384 // N), 16
            bits = si.make_qkv(B, H, N, d, seed=0)
            q, k, v = (torch.from_numpy(b.view(np.int16)).view(torch.bfloat16).cuda() for b in bits)
            o = torch.empty_like(q)
            lse = torch.empty((B, H, N), dtype=torch.float32, device="cuda")
            res = {}
            for c in (False, True):
                run = lambda: fa.fa_fwd(q, k, v, causal=c, out=o, lse=lse)
                for _ in range(args.warmup):
                    run()
                ms, clk = _event_loop(run, args.steps)
                tf = flops(B, H, N, d, c) / (ms / 1e3) / 1e12
                res["causal" if c else "non_causal"] = {
                    "ms_per_launch": ms, "tflops": tf, "frac_of_measured_burst": tf / peaks["bf16"],
                    "tflops_per_ghz": tf / (clk["sm_mhz"] / 1e3) if clk.get("sm_mhz") else None,
                    "clocks": clk, "schedule": schedule_of(N, d, c)}
            print(json.dumps({"suite": "sweep", "metric": METRIC, "unit": "TFLOP/s", "B": B, "H": H,
                              "N": N, "d": d, "dtype": "bf16", "data": "synthetic N(0,1), seed 0",
                              "steps": args.steps, "warmup": args.warmup, "modes": res,
                              "peak": peaks["bf16"], "impl": "ours"}), flush=True)
            del q, k, v, o, lse
            torch.cuda.empty_cache()


def bench_rescale(args):
    """The cost of the lazy O rescale on the headline shape (B=1, H=32, N=16384,
    d=128): for q, k ~ N(0, sigma^2) with sigma in {1, sqrt(3), 3}, both masks,
    the table's schedule (or --schedule) is timed like the headline (--warmup,
    then --steps launches, clocks sampled) and run once more with the rescale
    counters on (fa_fwd_rescale_stats): one JSON line per (sigma, mask) with
    TFLOP/s, TFLOP/s per GHz and the share of (warp, key tile) and (row, key
    tile) steps that rescaled O."""
    import numpy as np
    import torch
    import attention_forward_17_b200 as fa
    import seeded_inputs as si
    B, H, N, d = 1, 32, 16384, 128
    for sigma in (1.0, 3.0 ** 0.5, 3.0):
        bits = si.make_qkv(B, H, N, d, seed=0, sigma_qk=sigma)
        q, k, v = (torch.from_numpy(b.view(np.int16)).view(torch.bfloat16).cuda() for b in bits)
        o = torch.empty_like(q)
        lse = torch.empty((B, H, N), dtype=torch.float32, device="cuda")
        for c in (False, True):
            kw = {} if args.schedule is None else {"schedule": args.schedule}
            run = lambda: fa.fa_fwd(q, k, v, causal=c, out=o, lse=lse, **kw)
            for _ in range(args.warmup):
                run()
            ms, clk = _event_loop(run, args.steps)
            tf = flops(B, H, N, d, c) / (ms / 1e3) / 1e12
            _, _, w, r, total = fa.rescale_stats(q, k, v, c, schedule=args.schedule)
            print(json.dumps({"suite": "rescale", "B": B, "H": H, "N": N, "d": d, "qk_sigma": sigma,
                              "mode": "causal" if c else "non-causal",
                              "schedule": schedule_of(N, d, c, args.schedule), "tflops": tf,
                              "tflops_per_ghz": tf / (clk["sm_mhz"] / 1e3) if clk.get("sm_mhz") else None,
                              "clocks": clk, "warp_steps_rescaled": w, "row_steps_rescaled": r,
                              "warp_steps": total, "warp_step_rate": w / total,
                              "row_step_rate": r / (32 * total), "steps": args.steps,
                              "warmup": args.warmup, "impl": "ours"}), flush=True)
        del q, k, v, o, lse
        torch.cuda.empty_cache()


def main():
    ap = argparse.ArgumentParser(description=__doc__.split("\n")[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--suite", choices=["attention", "next", "sweep", "rescale"], default="attention",
                    help="'next' measures the kernels beyond the attention path, one line each; "
                         "'sweep' the sequence-length sweep, one line per (d, N); 'rescale' the "
                         "lazy-rescale rate and its cost against the score range")
    ap.add_argument("--next", nargs="+", choices=["row_softmax", "gemm", "vector_add"],
                    default=["row_softmax", "gemm", "vector_add"],
                    help="kernels measured by --suite next")
    ap.add_argument("--workload", choices=sorted(WORKLOADS), default=DEFAULT_WORKLOAD)
    ap.add_argument("--modes", choices=sorted(MODES), default="both",
                    help="masking modes in one step (the headline uses both)")
    ap.add_argument("--schedule", type=int, default=None,
                    help="pin the attention kernel schedule id (default: the search table's choice)")
    ap.add_argument("--causal-group", type=int, default=None,
                    help="pin the causal launch group (default: the search table's choice)")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-context", action="store_true",
                    help="skip the torch SDPA context timing")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-seconds", type=float, default=12.0,
                    help="target CPU time of the oracle sample")
    ap.add_argument("--ref-rows", type=int, default=64,
                    help="query rows per step of the reference (oracle) arm")
    args = ap.parse_args()
    if args.warmup < 3:
        raise SystemExit("--warmup must be >= 3")
    cfg = WORKLOADS[args.workload]
    if args.suite == "sweep":
        bench_sweep(args)
        return
    if args.suite == "rescale":
        bench_rescale(args)
        return
    if args.suite == "next":
        for name in args.next:
            {"row_softmax": bench_row_softmax, "gemm": bench_gemm,
             "vector_add": bench_vector_add}[name](args)
        return
    if args.impl == "reference":
        run_reference(args, cfg)
    else:
        run_ours(args, cfg)


if __name__ == "__main__":
    main()
