"""CPU checks of bench.py's measurement helpers: the FLOP convention, the
hash-gated DRAM traffic lookups, the clock-sample summary and the schedule
report."""
import hashlib
import os

import pytest

import bench


def test_flop_convention():
    # 4*B*H*N^2*d non-causal, exactly half of that causal
    assert bench.flops(1, 32, 16384, 128, False) == 4.0 * 32 * 16384 ** 2 * 128
    assert bench.flops(2, 16, 4096, 128, True) == 0.5 * bench.flops(2, 16, 4096, 128, False)


def test_profile_traffic_is_gated_by_the_source_hash(tmp_path, monkeypatch):
    src = tmp_path / "k.cuh"
    src.write_bytes(b"kernel v1")
    h = hashlib.sha256(b"kernel v1").hexdigest()[:16]
    (tmp_path / "profiles").mkdir()
    (tmp_path / "profiles" / "p.md").write_text(
        f"kernel_source_sha256_16: {h}\ntraffic_bytes_per_launch: 1.5e9\n")
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    assert bench.profile_traffic("p.md", "k.cuh") == 1.5e9
    src.write_bytes(b"kernel v2")                     # the kernel changed since the capture
    assert bench.profile_traffic("p.md", "k.cuh") is None
    assert bench.profile_traffic("missing.md", "k.cuh") is None


def test_headline_traffic_follows_the_kernel_family():
    # each kernel family reads its own summary; the figure is reported while the
    # summary's source hash matches the kernel, and withheld (with the reason) after
    for alg, name in ((0, "fa_fwd_kernel"), (1, "fa_fwd_pp_kernel"), (2, "fa_fwd_2q_kernel")):
        val, why = bench.measured_traffic(bench.DEFAULT_WORKLOAD, alg)
        prof = os.path.join(bench.ROOT, "profiles", f"{name}_b1_h64_n4096_d128_ncu.md")
        if val is not None:
            assert val > 0 and name in why
        elif os.path.exists(prof):
            assert why == "kernel changed since the ncu capture"
        else:
            assert why is None          # no capture of this kernel family committed
    # other workloads are not covered by the profiling capture
    assert bench.measured_traffic("b2_h16_n4096_d128", 0) == (None, None)


def test_clock_summary_uses_loaded_samples():
    c = bench.ClockSampler(0)
    c.source = "test"
    c.rows = [dict(sm=1965.0, smax=1965.0, power=120.0, reasons=set()),          # idle: ignored
              dict(sm=1600.0, smax=1965.0, power=900.0, reasons={"sw_power_cap"}),
              dict(sm=1500.0, smax=1965.0, power=980.0, reasons={"sw_power_cap"}),
              dict(sm=1700.0, smax=1965.0, power=700.0, reasons=set())]
    s = c.summary()
    assert s["sm_mhz"] == 1600.0 and s["samples"] == 3 and s["sm_max_mhz"] == 1965.0
    assert s["reasons"] == ["sw_power_cap"] and s["power_w_max"] == 980.0


def test_clock_summary_without_samples():
    c = bench.ClockSampler(0)
    assert c.summary()["sm_mhz"] is None


def test_schedule_report_respects_pins():
    auto = bench.schedule_of(16384, 128, True)
    pinned = bench.schedule_of(16384, 128, True, schedule=0, causal_group=3)
    assert pinned["id"] == 0 and pinned["causal_group"] == 3
    assert auto["id"] >= 0 and "algorithm" in auto
    assert bench.schedule_of(4096, 64, False)["causal_group"] is None


def test_sample_parity_checks_all_three_bars():
    import numpy as np
    import torch
    rng = np.random.default_rng(0)
    d, n = 8, 40
    o_ref = rng.standard_normal((n, d))
    lse_ref = rng.standard_normal(n)
    rows = np.arange(n)
    o = torch.tensor(o_ref, dtype=torch.float32).to(torch.bfloat16).view(1, 1, n, d)
    lse = torch.tensor(lse_ref, dtype=torch.float32).view(1, 1, n)
    res = [(rows, {False: (o_ref, lse_ref)})]
    good = bench.sample_parity(res, {False: o}, {False: lse}, d)
    assert good["pass"] and good["o_rel_l2"] < 1e-2
    # a uniform 1.5 % relative error stays under the max-abs bar (|O| <= ~1.3 here)
    # but fails the relative-L2 bar
    far = torch.tensor(o_ref * 1.015, dtype=torch.float32).view(1, 1, n, d)
    o_ref_small = o_ref * (0.01 / np.abs(o_ref).max())
    res_small = [(rows, {False: (o_ref_small, lse_ref)})]
    bad = bench.sample_parity(res_small, {False: torch.tensor(o_ref_small * 1.015).view(1, 1, n, d)},
                              {False: lse}, d)
    assert bad["o_max_abs"] <= 2e-2 and bad["o_rel_l2"] > 1e-2 and not bad["pass"]
    assert not bench.sample_parity(res, {False: far}, {False: lse + 0.01}, d)["pass"]
