"""Every compiled schedule of the attention kernel against the fp64 oracle
(ragged N, both masking modes, wide score range), the causal launch groups
(including a group size that does not divide B*H, so the last group is
partial: a tile launched twice or never would show), the persistent launch
with several tiles per CTA, and the table's choice for each problem class."""
import numpy as np
import pytest

import attention_forward_17_b200 as fa_lib
import oracle
import parity_utils as pu

pytestmark = pytest.mark.gpu

# the library loads without a GPU, so the compiled schedules are known at collection
N_SCHEDULES = fa_lib.lib.fa_schedule_count()


def _schedules():
    return fa_lib.schedules()


def run_sched(qt, kt, vt, causal, sid, group):
    import torch
    import attention_forward_17_b200 as fa
    o, lse = fa.fa_fwd(qt, kt, vt, causal, schedule=sid, causal_group=group)
    torch.cuda.synchronize()
    return pu.o_f64(o), lse.double().cpu().numpy()


@pytest.mark.parametrize("sid", range(N_SCHEDULES))
def test_every_schedule_matches_oracle(cuda_device, sid):
    sched = _schedules()
    d = sched[sid]["d"]
    (q, k, v), (qt, kt, vt) = pu.inputs(1, 2, 1000, d, seed=sid, sigma_qk=3.0)
    for causal in (False, True):
        o_ref, lse_ref = oracle.attention_fwd(q, k, v, causal, pu.default_scale(d))
        o, lse = run_sched(qt, kt, vt, causal, sid, 1)
        pu.check(o, lse, o_ref, lse_ref, f"schedule {sched[sid]} causal={causal}")


@pytest.mark.parametrize("group", [1, 2, 3, 5, 64])
def test_causal_groups_cover_every_tile(cuda_device, group):
    # B*H = 5 slices of 5 query tiles (N = 600, last tile ragged)
    (q, k, v), (qt, kt, vt) = pu.inputs(1, 5, 600, 64, seed=group)
    o_ref, lse_ref = oracle.attention_fwd(q, k, v, True, pu.default_scale(64))
    for s in _schedules():
        if s["d"] == 64 and s["persistent"] != 1 and s["emu_every"] == 4:   # forms that use the group
            o, lse = run_sched(qt, kt, vt, True, s["id"], group)
            pu.check(o, lse, o_ref, lse_ref, f"group {group} schedule {s}")


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("N", [1000, 1100])
def test_persistent_walks_every_tile(cuda_device, d, N):
    # 64 slices x 8 or 9 query tiles on 148 SMs: each persistent CTA takes
    # several tiles (non-causal) or several two-tile units (causal; N = 1100
    # gives an odd tile count, so the middle tile of each slice stands alone);
    # with cluster launch control, CTAs take over the tiles of CTAs that had not
    # launched yet
    sched = [s for s in _schedules() if s["d"] == d and s["persistent"]]
    assert sched, "no persistent schedule compiled"
    (q, k, v), (qt, kt, vt) = pu.inputs(1, 64, N, d, seed=N + d)
    for causal in (False, True):
        o_ref, lse_ref = oracle.attention_fwd(q, k, v, causal, pu.default_scale(d))
        for s in sched:
            o, lse = run_sched(qt, kt, vt, causal, s["id"], 1)
            pu.check(o, lse, o_ref, lse_ref, f"persistent {s} causal={causal} N={N}")


@pytest.mark.gpu
def test_two_tile_kernel_edges(cuda_device):
    # the multi-tile kernel on shapes that exercise its grouping of query tiles
    # (pairs, or triples): one row, a lone first tile, a group whose last tiles
    # are ragged or empty, several slices, both masks
    sched = [s for s in _schedules() if s["algorithm"] >= 2]
    assert sched, "no two-query-tile schedule compiled"
    for s in sched:
        d = s["d"]
        for B, H, N in ((1, 1, 1), (1, 2, 100), (1, 1, 129), (2, 1, 255), (1, 3, 256), (1, 2, 257),
                        (1, 1, 385), (2, 2, 640)):
            (q, k, v), (qt, kt, vt) = pu.inputs(B, H, N, d, seed=N + d, sigma_qk=3.0)
            for causal in (False, True):
                o_ref, lse_ref = oracle.attention_fwd(q, k, v, causal, pu.default_scale(d))
                o, lse = run_sched(qt, kt, vt, causal, s["id"], 1)
                pu.check(o, lse, o_ref, lse_ref, f"two-tile {s} B{B} H{H} N{N} causal={causal}")


def test_default_path_uses_the_table_choice(cuda_device):
    # fa_fwd (no schedule) and fa_fwd_schedule with the table's pick are the same launch
    import torch
    import attention_forward_17_b200 as fa
    (_, _, _), (qt, kt, vt) = pu.inputs(2, 3, 700, 128, seed=4)
    for causal in (False, True):
        sid, grp = fa.pick_schedule(700, 128, causal)
        o1, l1 = fa.fa_fwd(qt, kt, vt, causal)
        o2, l2 = fa.fa_fwd(qt, kt, vt, causal, schedule=sid, causal_group=grp)
        torch.cuda.synchronize()
        assert torch.equal(o1, o2) and torch.equal(l1, l2)
