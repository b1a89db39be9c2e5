"""Schedule search for the attention kernel (the TileLang tutorial's
autotuning step: define a search space, filter it by the on-chip budget,
benchmark and validate every candidate, cache the winner).

The search space is what libfa_b200.so has compiled (``schedules()``): the
share of exponentials evaluated by polynomial on the FMA pipe (none, 1/4, 1/2)
times the depth of the K/V shared-memory ring, the split-KV ping-pong
variant of the kernel (two softmax warp groups on alternate key tiles), plus
two persistent launch
forms (one CTA per SM walking several query tiles; or one CTA per tile whose
running CTAs take over the tiles of unlaunched ones by cluster launch
control), each instantiation already filtered at compile time to fit 227 KiB
of shared memory and 512 TMEM columns.  Under the causal mask the launch-group
size (heads whose query tiles are launched longest-first together) is searched
as well, for the launch forms that follow the grid order.

For every head dimension, masking mode and sequence-length bucket the script
times each candidate on a B200 (CUDA events, inputs larger than L2), checks
its output against the default schedule's (the default is the one the parity
tests pin to the fp64 oracle; the test suite also runs every schedule against
the oracle), and writes the fastest into ``csrc/fa_schedule_table.h``.  A
candidate replaces the default only if it is more than 1 % faster.  For the
longest sequences, which run at the power cap in practice, the default and the
fastest burst candidates are re-timed under sustained load on wide-range
scores (q, k ~ N(0, 3^2), the case that exercises the online rescaling) and
that decides.  Each
candidate is timed in three rounds that start at different candidates, and its
best round counts, so power-cap clock drift during the search does not favour
whichever candidate is timed first.

    python -m attention_forward_17_b200.schedule_search            # print the results
    python -m attention_forward_17_b200.schedule_search --write    # also rewrite the table
    python -m attention_forward_17_b200.schedule_search --report FILE.md
"""
from __future__ import annotations

import argparse
import datetime
import os
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
TABLE = os.path.join(HERE, "csrc", "fa_schedule_table.h")

# (N timed, largest N of the bucket it stands for); problem size B*H*N = 16 * 16384
BUCKETS = [(1024, 2048), (4096, 8192), (16384, None)]
GROUPS = [1, 2, 4, 8, 16]
MARGIN = 1.01
REPS = 3
SUSTAINED_FROM_N = 16384   # buckets decided under sustained load
FINALISTS = 2
SOAK_S = 0.3
SUSTAINED_SIGMA = 3.0


def _inputs(N, d, sigma_qk=1.0):
    import numpy as np
    import torch
    if ROOT not in sys.path:
        sys.path.insert(0, ROOT)
    import seeded_inputs as si
    B, H = max(1, 16384 // N), 16
    q, k, v = si.make_qkv(B, H, N, d, seed=0, sigma_qk=sigma_qk)
    dev = lambda x: torch.from_numpy(x.view(np.int16)).view(torch.bfloat16).cuda()
    return dev(q), dev(k), dev(v)


def _time(fn, warmup=3, iters=10):
    import torch
    for _ in range(warmup):
        fn()
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize()
    a.record()
    for _ in range(iters):
        fn()
    b.record()
    torch.cuda.synchronize()
    return a.elapsed_time(b) / iters


def _soak(fn, seconds):
    """Launch fn back to back for about `seconds` (untimed) so the GPU reaches its
    sustained clock under the power cap."""
    import time
    import torch
    t0 = time.perf_counter()
    while time.perf_counter() - t0 < seconds:
        for _ in range(8):
            fn()
        torch.cuda.synchronize()


def search(log=print):
    import torch
    from . import _binding as fa
    sustained = []   # (d, causal, N, schedule, group, burst tflops, sustained tflops)
    rows = []        # (d, causal, N, schedule, group, tflops, ok)
    table = []       # (d, causal, n_max, emu, slots, group)
    all_sched = fa.schedules()
    for d in (128, 64):
        cands = [s for s in all_sched if s["d"] == d]
        default = cands[0]
        for causal in (False, True):
            for N, n_max in BUCKETS:
                q, k, v = _inputs(N, d)
                B, H = q.shape[0], q.shape[1]
                flop = 4.0 * B * H * N * N * d / (2 if causal else 1)
                ref_o, ref_l = fa.fa_fwd(q, k, v, causal, schedule=default["id"], causal_group=1)
                torch.cuda.synchronize()
                o = torch.empty_like(ref_o)
                lse = torch.empty_like(ref_l)
                groups = [g for g in GROUPS if g <= B * H] if causal else [1]
                cand = [(s, g) for s in cands for g in (groups if s["persistent"] != 1 else [1])]
                # validate each candidate once against the default schedule's output
                valid = []
                for s, g in cand:
                    fa.fa_fwd(q, k, v, causal, out=o, lse=lse, schedule=s["id"], causal_group=g)
                    torch.cuda.synchronize()
                    do = (o.float() - ref_o.float()).abs().max().item()
                    dl = (lse - ref_l).abs().max().item()
                    rel = ((o.float() - ref_o.float()).norm() / ref_o.float().norm()).item()
                    ok = do <= 2e-2 and dl <= 1e-3 and rel <= 1e-2 and bool(torch.isfinite(o.float()).all())
                    valid.append((ok, do, dl))
                # time them REPS times, each round starting at a different candidate,
                # and keep each candidate's best round: the clock drops as the GPU
                # heats towards its power cap, and a fixed order would favour
                # whichever candidate always runs first
                best_tf = [0.0] * len(cand)
                for rep in range(REPS):
                    start = rep * len(cand) // REPS
                    for idx in list(range(start, len(cand))) + list(range(start)):
                        s, g = cand[idx]
                        ms = _time(lambda: fa.fa_fwd(q, k, v, causal, out=o, lse=lse,
                                                     schedule=s["id"], causal_group=g))
                        best_tf[idx] = max(best_tf[idx], flop / (ms / 1e3) / 1e12)
                results = []
                for (s, g), tf, (ok, do, dl) in zip(cand, best_tf, valid):
                    results.append((s, g, tf, ok))
                    rows.append((d, causal, N, s, g, tf, ok, do, dl))
                    log(f"d={d} causal={int(causal)} N={N:5d} emu={s['emu_every']} "
                        f"slots={s['kv_slots']} persist={s['persistent']} alg={s['algorithm']} "
                        f"group={g:2d}  "
                        f"{tf:7.1f} TFLOP/s  "
                        f"{'ok' if ok else 'REJECTED'} (|dO|={do:.2e}, |dLSE|={dl:.2e})")
                base = [r for r in results if r[0]["id"] == default["id"] and r[1] == 1][0]
                if N >= SUSTAINED_FROM_N:
                    # long sequences run at the power cap in practice: re-time the default and
                    # the fastest burst candidates under sustained load and decide on that
                    # finalists: the default, the fastest burst candidate of every launch form
                    # and algorithm, and the two fastest overall
                    ok_rs = sorted((r for r in results if r[3]), key=lambda r: -r[2])
                    finalists = [base]
                    classes = {(r[0]["persistent"], r[0]["algorithm"]) for r in ok_rs}
                    picks = [next(r for r in ok_rs if (r[0]["persistent"], r[0]["algorithm"]) == cl)
                             for cl in sorted(classes)] + ok_rs[:FINALISTS]
                    for r in picks:
                        if all(r is not f for f in finalists):
                            finalists.append(r)
                    # decided on the wide score range (q, k ~ N(0, 3^2)), where the online
                    # rescaling is exercised hardest
                    q, k, v = _inputs(N, d, SUSTAINED_SIGMA)
                    sus = [0.0] * len(finalists)
                    for rep in range(REPS):
                        start = rep * len(finalists) // REPS
                        for idx in list(range(start, len(finalists))) + list(range(start)):
                            s, g, _, _ = finalists[idx]
                            f = lambda: fa.fa_fwd(q, k, v, causal, out=o, lse=lse, schedule=s["id"],
                                                  causal_group=g)
                            _soak(f, SOAK_S)
                            sus[idx] = max(sus[idx], flop / (_time(f, warmup=0, iters=20) / 1e3) / 1e12)
                    for (s, g, tf, _), st in zip(finalists, sus):
                        sustained.append((d, causal, N, s, g, tf, st))
                        log(f"   sustained: emu={s['emu_every']} slots={s['kv_slots']} "
                            f"persist={s['persistent']} alg={s['algorithm']} group={g:2d}  {st:7.1f} TFLOP/s")
                    top = max(range(len(finalists)), key=lambda i: sus[i])
                    if sus[top] < sus[0] * MARGIN:
                        top = 0
                    best = (finalists[top][0], finalists[top][1], sus[top], True)
                    base = (base[0], base[1], sus[0], True)
                else:
                    best = max((r for r in results if r[3]), key=lambda r: r[2])
                    if best[2] < base[2] * MARGIN:
                        best = base
                table.append((d, int(causal), n_max, best[0]["emu_every"], best[0]["kv_slots"], best[1],
                              best[0]["persistent"], best[0]["algorithm"]))
                log(f"  -> d={d} causal={int(causal)} N<={n_max or 'max'}: emu={best[0]['emu_every']} "
                    f"slots={best[0]['kv_slots']} persist={best[0]['persistent']} "
                    f"alg={best[0]['algorithm']} group={best[1]} "
                    f"({best[2]:.1f} vs default {base[2]:.1f} TFLOP/s)")
                del q, k, v, o, lse, ref_o, ref_l
                torch.cuda.empty_cache()
    return rows, table, sustained


def write_table(table, device_name, path=TABLE):
    stamp = datetime.date.today().isoformat()
    lines = [
        "// Schedule table of the attention kernel: for each head dimension, masking",
        "// mode and sequence-length bucket (N <= n_max), the exponential split, the",
        "// K/V ring depth, the causal launch group, the launch form and the algorithm.  Written by",
        f"// attention_forward_17_b200/schedule_search.py on {device_name} ({stamp}).",
        "#pragma once",
        "",
        "#include <cstdint>",
        "",
        "namespace fa {",
        "",
        "struct ScheduleTableEntry {",
        "    int d;",
        "    int causal;",
        "    int64_t n_max;",
        "    int emu;",
        "    int slots;",
        "    int group;",
        "    int persist;",
        "    int alg;",
        "};",
        "",
        "constexpr ScheduleTableEntry kScheduleTable[] = {",
    ]
    for d, causal, n_max, emu, slots, group, persist, alg in table:
        nm = "INT64_MAX" if n_max is None else str(n_max)
        lines.append(f"    {{{d}, {causal}, {nm}, {emu}, {slots}, {group}, {persist}, {alg}}},")
    lines += ["};", "", "}  // namespace fa", ""]
    with open(path, "w") as f:
        f.write("\n".join(lines))


def write_report(rows, table, device_name, path, top=5, sustained=()):
    """Markdown summary: per (d, causal, N) the default schedule and the `top`
    fastest candidates, then the chosen table."""
    cmd = "python -m attention_forward_17_b200.schedule_search --write --report " + os.path.relpath(path, ROOT)
    out = [f"# Attention schedule search on {device_name}", "",
           "Command (repository root, one GPU):", "", f"    {cmd}", "",
           "B = 16384 / N, H = 16, bf16 N(0,1), seed 0; TFLOP/s by the 4*B*H*N^2*d (non-causal) / half "
           "(causal) convention; per candidate the best of 3 rounds (rotated order) of 3 warm-up + 10 timed "
           "launches, CUDA events. `ok` = output within the parity tolerances of the default schedule's. "
           "launch: 0 one CTA per tile, 1 static persistent, 2 cluster launch control; alg: 0 standard, "
           "1 split-KV ping-pong. Per problem: the default and the fastest candidates.", ""]
    keys = []
    for r in rows:
        if (r[0], r[1], r[2]) not in keys:
            keys.append((r[0], r[1], r[2]))
    for d, causal, N in keys:
        rs = [r for r in rows if (r[0], r[1], r[2]) == (d, causal, N)]
        default = rs[0]
        best = sorted(rs, key=lambda r: -r[5])[:top]
        out += [f"**d={d} {'causal' if causal else 'non-causal'} N={N}** ({len(rs)} candidates)", "",
                "| emu | slots | launch | alg | group | TFLOP/s | ok |", "|---|---|---|---|---|---|---|"]
        for r in [default] + [b for b in best if b is not default]:
            _, _, _, sch, g, tf, ok, _, _ = r
            tag = " (default)" if r is default else ""
            out.append(f"| {sch['emu_every']} | {sch['kv_slots']} | {sch['persistent']} | "
                       f"{sch['algorithm']} | {g} | {tf:.1f}{tag} | {'yes' if ok else 'no'} |")
        rejected = [r for r in rs if not r[6]]
        if rejected:
            out.append(f"\n{len(rejected)} candidate(s) rejected by the output check.")
        out.append("")
    if sustained:
        out += [f"Sustained load (N >= {SUSTAINED_FROM_N}: the default, the fastest burst candidate of "
                f"each launch form and algorithm and the {FINALISTS} fastest overall, on q, k ~ N(0, "
                f"{SUSTAINED_SIGMA:g}^2) inputs, each launched back to back for {SOAK_S} s before 20 timed "
                f"launches, best of {REPS} rotated rounds; these decide the bucket; `burst` is the sigma = 1 "
                f"burst figure):", "",
                "| d | causal | N | emu | slots | launch | alg | group | burst | sustained |",
                "|---|---|---|---|---|---|---|---|---|---|"]
        for d, causal, N, sch, g, tf, st in sustained:
            out.append(f"| {d} | {int(causal)} | {N} | {sch['emu_every']} | {sch['kv_slots']} | "
                       f"{sch['persistent']} | {sch['algorithm']} | {g} | {tf:.1f} | {st:.1f} |")
        out.append("")
    out += ["Chosen (table written to `attention_forward_17_b200/csrc/fa_schedule_table.h`):", "",
            "| d | causal | N <= | emu | slots | group | launch | alg |", "|---|---|---|---|---|---|---|---|"]
    for d, causal, n_max, emu, slots, group, persist, alg in table:
        out.append(f"| {d} | {causal} | {n_max or 'any'} | {emu} | {slots} | {group} | {persist} | {alg} |")
    with open(path, "w") as f:
        f.write("\n".join(out) + "\n")


def main():
    ap = argparse.ArgumentParser(description=__doc__.split("\n")[0])
    ap.add_argument("--write", action="store_true", help="rewrite csrc/fa_schedule_table.h")
    ap.add_argument("--report", default=None, help="write a markdown report of every timing")
    args = ap.parse_args()
    import torch
    name = torch.cuda.get_device_name(0)
    rows, table, sustained = search()
    if args.write:
        write_table(table, name)
        print(f"wrote {TABLE}")
    if args.report:
        write_report(rows, table, name, args.report, sustained=sustained)
        print(f"wrote {args.report}")


if __name__ == "__main__":
    main()
