"""Schedule search for the attention kernel (the TileLang tutorial's
autotuning step: define a search space, filter it by the on-chip budget,
benchmark and validate every candidate, cache the winner).

The search space is what libfa_b200.so has compiled (``schedules()``): the
algorithm (one query tile per CTA; the split-KV ping-pong variant with two
softmax groups on alternate key tiles; two query tiles per CTA with P kept in
tensor memory), the share of exponentials evaluated by polynomial on the FMA
pipe, the depth of the K/V shared-memory ring, the key-tile rows of the
two-tile kernel (64, 128, 192 where tensor memory allows) and, for the
one-tile kernel,
the launch form (one CTA per tile; a persistent CTA per SM walking several
tiles; or one CTA per tile whose running CTAs take over the tiles of
unlaunched ones by cluster launch control), each instantiation already
filtered at compile time to fit 227 KiB of shared memory and 512 TMEM columns.
Under the causal mask the launch-group size (heads whose query tiles are
launched longest-first together) is searched as well, for the launch forms
that follow the grid order.

Every candidate is timed the way the benchmark times the headline: 5 warm-up
launches, then 20 launches between CUDA events, with the SM clock, power and
clock-event reasons sampled during the timed launches (``clocks.py``); each
point reports TFLOP/s, the median SM clock and TFLOP/s per GHz.  Candidates are
timed in three rounds that start at different candidates and keep their best
round, so the drift of the clock as the GPU approaches its power cap does not
favour whichever candidate is timed first.  Each candidate's output is first
checked against the default schedule's (the parity tests pin every schedule
to the fp64 oracle; two outputs that each meet the oracle's bars can differ by
up to twice them, which is the bound used here).  A candidate replaces the
default only if it is more than
1 % faster.  Buckets and their timed problem (N B H = 16 * 16384 query rows):

    N <= 2048   N = 1024,  B = 16, H = 16, q, k ~ N(0, 1)
    N <= 8192   N = 4096,  B = 4,  H = 16, q, k ~ N(0, 1)
    N >  8192   N = 16384, B = 1,  H = 32, q, k ~ N(0, 3^2): the headline
                workload itself, so the table's choice for it is made on the
                benchmark's own inputs and timing.

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

# (N timed, largest N of the bucket, B, H, sigma of q and k)
BUCKETS = [(1024, 2048, 16, 16, 1.0), (4096, 8192, 4, 16, 1.0), (16384, None, 1, 32, 3.0)]
GROUPS = [1, 4, 16]
MARGIN = 1.01
REPS = 3
WARMUP, ITERS = 5, 20


def _inputs(B, H, N, d, sigma_qk):
    import numpy as np
    import torch
    if ROOT not in sys.path:
        sys.path.insert(0, ROOT)
    import seeded_inputs as si
    q, k, v = si.make_qkv(B, H, N, d, seed=0, sigma_qk=sigma_qk)
    dev = lambda x: torch.from_numpy(x.view(np.int16)).view(torch.bfloat16).cuda()
    return dev(q), dev(k), dev(v)


def _time(fn):
    """Mean ms of ITERS launches after WARMUP, CUDA events, clocks sampled meanwhile."""
    import torch
    from .clocks import ClockSampler
    for _ in range(WARMUP):
        fn()
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize()
    with ClockSampler(torch.cuda.current_device()) as clk:
        a.record()
        for _ in range(ITERS):
            fn()
        b.record()
        torch.cuda.synchronize()
    return a.elapsed_time(b) / ITERS, clk.summary()


def _per_ghz(tf, clk):
    mhz = clk.get("sm_mhz")
    return tf / (mhz / 1e3) if mhz else None


def search(log=print):
    import torch
    from . import _binding as fa
    rows = []        # dicts: one per (problem, candidate)
    table = []       # (d, causal, n_max, emu, slots, group, persist, alg)
    all_sched = fa.schedules()
    for d in (128, 64):
        cands = [s for s in all_sched if s["d"] == d]
        default = cands[0]
        for causal in (False, True):
            for N, n_max, B, H, sigma in BUCKETS:
                q, k, v = _inputs(B, H, N, d, sigma)
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
                    # both outputs are held to the fp64 oracle's bars (2e-2 max-abs and
                    # 1e-2 rel-L2 on O, 1e-3 on LSE) by the parity tests; two outputs
                    # within those bars can differ by up to twice them (one bf16 step of
                    # an |O| >= 4 value is already 2^-5), so twice the bars here
                    ok = do <= 4e-2 and dl <= 2e-3 and rel <= 2e-2 and bool(torch.isfinite(o.float()).all())
                    valid.append((ok, do, dl))
                best = [(0.0, None)] * len(cand)
                for rep in range(REPS):
                    start = rep * len(cand) // REPS
                    for idx in list(range(start, len(cand))) + list(range(start)):
                        s, g = cand[idx]
                        ms, clk = _time(lambda: fa.fa_fwd(q, k, v, causal, out=o, lse=lse,
                                                          schedule=s["id"], causal_group=g))
                        tf = flop / (ms / 1e3) / 1e12
                        if tf > best[idx][0]:
                            best[idx] = (tf, clk)
                results = []
                for (s, g), (tf, clk), (ok, do, dl) in zip(cand, best, valid):
                    r = dict(d=d, causal=causal, N=N, B=B, H=H, sigma=sigma, sched=s, group=g,
                             tflops=tf, clocks=clk, per_ghz=_per_ghz(tf, clk), ok=ok, d_o=do, d_lse=dl)
                    results.append(r)
                    rows.append(r)
                    pg = r["per_ghz"]
                    log(f"d={d} causal={int(causal)} N={N:5d} alg={s['algorithm']} bn={s['key_tile']} emu={s['emu_every']} "
                        f"slots={s['kv_slots']} persist={s['persistent']} group={g:2d}  "
                        f"{tf:7.1f} TFLOP/s at {clk.get('sm_mhz')} MHz "
                        f"({'%.1f' % pg if pg else '-'} per GHz; {','.join(clk.get('reasons', [])) or '-'})  "
                        f"{'ok' if ok else 'REJECTED'} (|dO|={do:.2e}, |dLSE|={dl:.2e})")
                base = next(r for r in results if r["sched"]["id"] == default["id"] and r["group"] == 1)
                win = max((r for r in results if r["ok"]), key=lambda r: r["tflops"])
                if win["tflops"] < base["tflops"] * MARGIN:
                    win = base
                s = win["sched"]
                table.append((d, int(causal), n_max, s["emu_every"], s["kv_slots"], win["group"],
                              s["persistent"], s["algorithm"], s["key_tile"]))
                log(f"  -> d={d} causal={int(causal)} N<={n_max or 'max'}: alg={s['algorithm']} bn={s['key_tile']} "
                    f"emu={s['emu_every']} slots={s['kv_slots']} persist={s['persistent']} "
                    f"group={win['group']} ({win['tflops']:.1f} vs default {base['tflops']:.1f} TFLOP/s)")
                del q, k, v, o, lse, ref_o, ref_l
                torch.cuda.empty_cache()
    return rows, table


def write_table(table, device_name, path=TABLE):
    stamp = datetime.date.today().isoformat()
    lines = [
        "// Schedule table of the attention kernel: for each head dimension, masking",
        "// mode and sequence-length bucket (N <= n_max), the exponential split, the",
        "// K/V ring depth, the causal launch group, the launch form, the algorithm and",
        "// the key-tile rows.  Written by",
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
        "    int bn;",
        "};",
        "",
        "constexpr ScheduleTableEntry kScheduleTable[] = {",
    ]
    for d, causal, n_max, emu, slots, group, persist, alg, bn in table:
        nm = "INT64_MAX" if n_max is None else str(n_max)
        lines.append(f"    {{{d}, {causal}, {nm}, {emu}, {slots}, {group}, {persist}, {alg}, {bn}}},")
    lines += ["};", "", "}  // namespace fa", ""]
    with open(path, "w") as f:
        f.write("\n".join(lines))


def write_report(rows, table, device_name, path, top=6):
    """Markdown summary: per (d, causal, N) the default schedule and the `top`
    fastest candidates with their clock records, then the chosen table."""
    cmd = "python -m attention_forward_17_b200.schedule_search --write --report " + os.path.relpath(path, ROOT)
    out = [f"# Attention schedule search on {device_name}", "",
           "Command (repository root, one GPU):", "", f"    {cmd}", "",
           "Per bucket the timed problem is N, B = 16384/N (1 at N = 16384), H = 16 (32 at N = 16384), "
           "bf16, seed 0, q, k ~ N(0, 1) (N(0, 3^2) at N = 16384: the headline workload). TFLOP/s by the "
           "4*B*H*N^2*d (non-causal) / half (causal) convention; per candidate the best of 3 rounds "
           f"(rotated order) of {WARMUP} warm-up + {ITERS} timed launches (CUDA events), the way the "
           "benchmark times the headline; MHz = median SM clock sampled (NVML, 10 ms) during that "
           "round's timed launches; per GHz = TFLOP/s / (MHz / 1000); reasons = clock-event reasons "
           "seen. `ok` = output within twice the oracle's parity bars of the default schedule's (each "
           "is held to the oracle's bars by the parity tests). alg: 0 one "
           "query tile per CTA, 1 split-KV ping-pong, 2 two query tiles per CTA, then + 1 two score buffers "
           "per tile, + 2 bf16 weight sums on the tensor core, + 4 P released as 3/4 and 1/4 of the keys, "
           "+ 8 three query tiles per CTA; launch: 0 one CTA "
           "per tile, 1 static persistent, 2 cluster launch control.", ""]
    keys = []
    for r in rows:
        if (r["d"], r["causal"], r["N"]) not in keys:
            keys.append((r["d"], r["causal"], r["N"]))
    for d, causal, N in keys:
        rs = [r for r in rows if (r["d"], r["causal"], r["N"]) == (d, causal, N)]
        default = rs[0]
        best = sorted(rs, key=lambda r: -r["tflops"])[:top]
        out += [f"**d={d} {'causal' if causal else 'non-causal'} N={N}** ({len(rs)} candidates)", "",
                "| alg | key tile | emu | slots | launch | group | TFLOP/s | MHz | per GHz | reasons | ok |",
                "|---|---|---|---|---|---|---|---|---|---|---|"]
        for r in [default] + [b for b in best if b is not default]:
            s, clk = r["sched"], r["clocks"] or {}
            tag = " (default)" if r is default else ""
            pg = r["per_ghz"]
            out.append(f"| {s['algorithm']} | {s['key_tile']} | {s['emu_every']} | {s['kv_slots']} | {s['persistent']} | "
                       f"{r['group']} | {r['tflops']:.1f}{tag} | {clk.get('sm_mhz')} | "
                       f"{'%.1f' % pg if pg else '-'} | {','.join(clk.get('reasons', [])) or '-'} | "
                       f"{'yes' if r['ok'] else 'no'} |")
        rejected = [r for r in rs if not r["ok"]]
        if rejected:
            out.append(f"\n{len(rejected)} candidate(s) rejected by the output check.")
        out.append("")
    out += ["Chosen (table written to `attention_forward_17_b200/csrc/fa_schedule_table.h`):", "",
            "| d | causal | N <= | emu | slots | group | launch | alg | key tile |",
            "|---|---|---|---|---|---|---|---|---|"]
    for d, causal, n_max, emu, slots, group, persist, alg, bn in table:
        out.append(f"| {d} | {causal} | {n_max or 'any'} | {emu} | {slots} | {group} | {persist} | {alg} | {bn} |")
    with open(path, "w") as f:
        f.write("\n".join(out) + "\n")


def main():
    ap = argparse.ArgumentParser(description=__doc__.split("\n")[0])
    ap.add_argument("--write", action="store_true", help="rewrite csrc/fa_schedule_table.h")
    ap.add_argument("--report", default=None, help="write a markdown report of every timing")
    args = ap.parse_args()
    import torch
    name = torch.cuda.get_device_name(0)
    rows, table = search()
    if args.write:
        write_table(table, name)
        print(f"wrote {TABLE}")
    if args.report:
        write_report(rows, table, name, args.report)
        print(f"wrote {args.report}")


if __name__ == "__main__":
    main()
