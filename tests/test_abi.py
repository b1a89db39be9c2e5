"""The C-ABI library loads on a machine without a GPU, exports every function
include/fa.h declares, and rejects bad arguments on the host, in the
documented order, before touching the device."""
import ctypes
import os
import subprocess

import pytest

import attention_forward_17_b200 as fa
from attention_forward_17_b200 import _binding as bnd

LIB = fa.lib


def test_exports_every_header_function():
    names = fa.header_functions()
    assert set(names) >= {"fa_fwd", "fa_fwd_status", "fa_fwd_host", "fa_strerror", "fa_version",
                          "fa_fwd_launches"}
    out = subprocess.run(["nm", "-D", "--defined-only", fa.LIB_PATH], capture_output=True,
                         text=True, check=True).stdout
    exported = {line.split()[-1] for line in out.splitlines() if line.strip()}
    for n in names:
        assert n in exported, f"{n} declared in include/fa.h but not exported"
        assert hasattr(LIB, n)


def test_no_torch_in_library():
    out = subprocess.run(["ldd", fa.LIB_PATH], capture_output=True, text=True).stdout
    assert "torch" not in out and "c10" not in out


def test_strerror_and_version():
    for code in range(-8, 1):
        s = fa.strerror(code)
        assert isinstance(s, str) and s
    assert fa.strerror(12345) == "unknown status"
    assert fa.version() == (1, 2)


def call(q=16, k=32, v=48, o=64, lse=80, B=1, H=1, N=128, d=64, causal=0, scale=0.125):
    # fake, never-dereferenced device addresses: every case below fails a host check first
    return LIB.fa_fwd(q, k, v, o, lse, B, H, N, d, causal, scale, None)


@pytest.mark.parametrize("kw,code", [
    (dict(B=-1), fa.FA_ERR_SHAPE),
    (dict(N=-5), fa.FA_ERR_SHAPE),
    (dict(q=0), fa.FA_ERR_NULL),
    (dict(lse=0), fa.FA_ERR_NULL),
    (dict(N=2 ** 31), fa.FA_ERR_SHAPE),
    (dict(B=2 ** 20, H=2 ** 12), fa.FA_ERR_SHAPE),
    (dict(d=96), fa.FA_ERR_HEADDIM),
    (dict(d=256), fa.FA_ERR_HEADDIM),
    (dict(q=18), fa.FA_ERR_ALIGN),
    (dict(o=72), fa.FA_ERR_ALIGN),
    (dict(lse=82), fa.FA_ERR_ALIGN),
    (dict(scale=0.0), fa.FA_ERR_SCALE),
    (dict(scale=-1.0), fa.FA_ERR_SCALE),
    (dict(scale=float("inf")), fa.FA_ERR_SCALE),
    (dict(scale=float("nan")), fa.FA_ERR_SCALE),
])
def test_argument_errors(kw, code):
    assert call(**kw) == code


def test_error_order():
    # shape before null before head-dim before alignment before scale
    assert call(B=-1, q=0) == fa.FA_ERR_SHAPE
    assert call(q=0, d=96) == fa.FA_ERR_NULL
    assert call(d=96, q=18) == fa.FA_ERR_HEADDIM
    assert call(q=18, scale=0.0) == fa.FA_ERR_ALIGN


@pytest.mark.parametrize("kw", [dict(B=0), dict(H=0), dict(N=0)])
def test_empty_problem_is_a_noop(kw):
    # pointers are not examined for an empty problem
    assert call(q=0, k=0, v=0, o=0, lse=0, d=96, **kw) == fa.FA_OK


def test_host_entry_checks():
    f = LIB.fa_fwd_host
    args = [1024, 2048, 3072, 4096, 5120, 16, 32, 48, 64, 80]
    bad = list(args)
    bad[0] = 0
    assert f(*bad, 1, 1, 128, 64, 0, 0.125, None) == fa.FA_ERR_NULL
    bad = list(args)
    bad[5] = 18
    assert f(*bad, 1, 1, 128, 64, 0, 0.125, None) == fa.FA_ERR_ALIGN
    assert f(*args, 1, 1, 0, 64, 0, 0.125, None) == fa.FA_OK


def test_selftest_argument_checks():
    assert LIB.fa_selftest_wait_timeout(None, 1000, 0, None) == fa.FA_ERR_NULL
    assert LIB.fa_selftest_wait_timeout(16, 0, 0, None) == fa.FA_ERR_SHAPE
    assert LIB.fa_selftest_wait_timeout(16, 10**8, 0, None) == fa.FA_ERR_SHAPE


def test_row_softmax_argument_checks():
    f = LIB.fa_row_softmax
    assert f(16, 32, -1, 8, 1.0, None) == fa.FA_ERR_SHAPE
    assert f(0, 0, 0, 8, 1.0, None) == fa.FA_OK
    assert f(0, 32, 4, 8, 1.0, None) == fa.FA_ERR_NULL
    assert f(17, 32, 4, 8, 1.0, None) == fa.FA_ERR_ALIGN
    assert f(16, 32, 4, 8, float("inf"), None) == fa.FA_ERR_SCALE
    assert f(16, 32, 2 ** 31, 8, 1.0, None) == fa.FA_ERR_SHAPE
    assert LIB.fa_row_softmax_launches(4, 8) == 1 and LIB.fa_row_softmax_launches(0, 8) == 0


def test_gemm_argument_checks():
    f = LIB.fa_gemm
    P, B_, G = fa.FA_GEMM_PLAIN, fa.FA_GEMM_BIAS, fa.FA_GEMM_BIAS_GELU
    assert f(16, 32, 48, 64, 8, 8, 8, 3, None, None) == fa.FA_ERR_ARG
    assert f(16, 32, 48, 64, 8, 8, 8, -1, None, None) == fa.FA_ERR_ARG
    assert f(16, 32, 48, 64, -1, 8, 8, G, None, None) == fa.FA_ERR_SHAPE
    assert f(16, 32, 48, 64, 8, 8, -8, G, None, None) == fa.FA_ERR_SHAPE
    assert f(None, None, None, None, 0, 8, 8, G, None, None) == fa.FA_OK      # empty: no-op
    assert f(None, None, None, None, 8, 0, 8, G, None, None) == fa.FA_OK
    assert f(16, 32, 48, None, 8, 8, 8, G, None, None) == fa.FA_ERR_NULL
    assert f(None, 32, 48, 64, 8, 8, 8, G, None, None) == fa.FA_ERR_NULL
    assert f(16, 32, None, 64, 8, 8, 8, B_, None, None) == fa.FA_ERR_NULL    # bias needed
    assert f(16, 32, 48, 64, 8, 12, 8, G, None, None) == fa.FA_ERR_SHAPE     # N % 8
    assert f(16, 32, 48, 64, 8, 8, 12, G, None, None) == fa.FA_ERR_SHAPE     # K % 8
    assert f(16, 32, 48, 64, 2 ** 31, 8, 8, G, None, None) == fa.FA_ERR_SHAPE
    assert f(18, 32, 48, 64, 8, 8, 8, G, None, None) == fa.FA_ERR_ALIGN
    assert f(16, 32, 50, 64, 8, 8, 8, G, None, None) == fa.FA_ERR_ALIGN
    assert f(16, 32, 48, 66, 8, 8, 8, G, None, None) == fa.FA_ERR_ALIGN
    # K = 0 needs neither A nor B; the plain epilogue needs no bias (checks then pass to the device)
    assert f(None, None, 48, 66, 8, 8, 0, G, None, None) == fa.FA_ERR_ALIGN
    assert f(16, 32, None, 66, 8, 8, 8, P, None, None) == fa.FA_ERR_ALIGN
    assert LIB.fa_gemm_launches(8, 8, 8) == 1 and LIB.fa_gemm_launches(0, 8, 8) == 0


def test_vector_add_argument_checks():
    f = LIB.fa_vector_add
    assert f(16, 32, 48, -1, None) == fa.FA_ERR_SHAPE
    assert f(None, None, None, 0, None) == fa.FA_OK
    assert f(None, 32, 48, 4, None) == fa.FA_ERR_NULL
    assert f(16, 32, 48, 2 ** 41, None) == fa.FA_ERR_SHAPE
    assert f(18, 32, 48, 4, None) == fa.FA_ERR_ALIGN
    assert LIB.fa_vector_add_launches(5) == 1 and LIB.fa_vector_add_launches(0) == 0


def test_schedule_registry():
    n = LIB.fa_schedule_count()
    assert n >= 2
    import ctypes
    vals = [ctypes.c_int() for _ in range(7)]
    seen = set()
    for i in range(n):
        assert LIB.fa_schedule_info(i, *[ctypes.byref(x) for x in vals]) == fa.FA_OK
        d, emu, slots, persist, alg, smem, bn = (x.value for x in vals)
        # key tiles of 128 rows, or 64 / 192 for the multi-tile kernel where the
        # score and output buffers of its query tiles fit the 512 TMEM columns
        # multi-tile algorithms: 2 + (1: two score buffers) + (2: l^ on the tensor core)
        # + (4: P released as three quarters and one quarter of the keys)
        # + (8: three query tiles per CTA instead of two)
        bits = alg - 2 if alg >= 2 else 0
        bufs = 2 if bits & 1 else 1           # score buffers per query tile
        do = d + 16 if bits & 2 else d        # O columns (16 more when the tensor core sums l^)
        nt = 3 if bits & 8 else 2             # query tiles per CTA
        assert nt * (bufs * bn + do) <= 512 and (bn == 128 or (alg >= 2 and bn in (64, 80, 192)))
        assert d in (64, 128) and emu in (0, 2, 3, 4, 8) and persist in (0, 1, 2)
        assert alg in range(18) and 0 < smem <= 232448
        assert not (bits & 4) or bn == 128     # the three-quarter release needs 128-row key tiles
        # the one-tile kernels need four slots for sound parity waits; the
        # two-tile kernel's issuers observe every load in order, so any depth >= 2
        assert slots >= (4 if alg < 2 or bits & 1 else 2)
        assert (d, emu, slots, persist, alg, bn) not in seen
        seen.add((d, emu, slots, persist, alg, bn))
    assert any(k[3] == 1 for k in seen) and any(k[3] == 2 for k in seen)
    assert any(k[4] == 1 for k in seen) and any(k[4] == 2 and k[0] == d for k in seen for d in (64, 128))
    assert {(k[0], k[5]) for k in seen} >= {(128, 64), (128, 128), (64, 64), (64, 128), (64, 192)}
    assert LIB.fa_schedule_info(n, None, None, None, None, None, None, None) == fa.FA_ERR_ARG
    assert LIB.fa_schedule_info(-1, None, None, None, None, None, None, None) == fa.FA_ERR_ARG
    # the first schedule of each head dimension is the default
    assert fa.schedules()[0]["d"] == 128


def test_schedule_argument_checks():
    f = LIB.fa_fwd_schedule
    args = (16, 32, 48, 64, 80, 1, 1, 128)
    n = LIB.fa_schedule_count()
    d64 = [s["id"] for s in fa.schedules() if s["d"] == 64][0]
    assert f(*args, 128, 0, 0.125, n, 1, None, None) == fa.FA_ERR_ARG     # unknown id
    assert f(*args, 128, 0, 0.125, d64, 1, None, None) == fa.FA_ERR_ARG   # id for another d
    assert f(*args, 128, 0, 0.125, -2, 1, None, None) == fa.FA_ERR_ARG
    assert f(*args, 128, 1, 0.125, 0, -1, None, None) == fa.FA_ERR_ARG
    # the attention arguments are checked first
    assert f(*args[:5], -1, 1, 128, 128, 0, 0.125, n, 1, None, None) == fa.FA_ERR_SHAPE
    assert f(*args[:5], 0, 1, 128, 128, 0, 0.125, n, 1, None, None) == fa.FA_OK
    assert f(*args, 96, 0, 0.125, 0, 1, None, None) == fa.FA_ERR_HEADDIM
    import ctypes
    sid, grp = ctypes.c_int(), ctypes.c_int()
    assert LIB.fa_fwd_pick_schedule(4096, 128, 1, ctypes.byref(sid), ctypes.byref(grp)) == fa.FA_OK
    assert LIB.fa_fwd_pick_schedule(4096, 128, 1, None, ctypes.byref(grp)) == fa.FA_ERR_NULL
    assert LIB.fa_fwd_pick_schedule(-1, 128, 1, ctypes.byref(sid), ctypes.byref(grp)) == fa.FA_ERR_SHAPE
    assert LIB.fa_fwd_pick_schedule(64, 80, 1, ctypes.byref(sid), ctypes.byref(grp)) == fa.FA_ERR_HEADDIM


def test_rescale_stats_argument_checks():
    f = LIB.fa_fwd_rescale_stats
    args = (16, 32, 48, 64, 80, 1, 1, 128, 128, 0, 0.125)
    assert f(*args, -1, None, None) == fa.FA_ERR_NULL          # counters required
    assert f(*args, -2, 96, None) == fa.FA_ERR_ARG             # schedule id below -1
    assert f(*args[:5], 0, 1, 128, 128, 0, 0.125, -1, None, None) == fa.FA_OK     # empty: no-op
    assert f(*args[:8], 80, 0, 0.125, -1, 96, None) == fa.FA_ERR_HEADDIM          # fa_fwd's checks first


def test_launch_count():
    assert fa.launches_per_call(1, 1, 128, 64) == 1
    assert fa.launches_per_call(0, 1, 128, 64) == 0


def test_binding_fails_loudly_without_library(tmp_path, monkeypatch):
    monkeypatch.setattr(bnd, "LIB_PATH", str(tmp_path / "missing.so"))
    with pytest.raises(ImportError):
        bnd._load()


def test_schedule_table_entries_are_compiled():
    # every row of the searched table must name a compiled schedule, or the
    # dispatch would silently fall back to the first schedule of that head dim
    import re
    import os
    path = os.path.join(os.path.dirname(fa.LIB_PATH), "csrc", "fa_schedule_table.h")
    rows = re.findall(r"\{(\d+), (\d), (\w+), (\d+), (\d+), (\d+), (\d), (\d+), (\d+)\},", open(path).read())
    assert rows, "no table rows parsed"
    compiled = {(s["d"], s["emu_every"], s["kv_slots"], s["persistent"], s["algorithm"], s["key_tile"])
                for s in fa.schedules()}
    buckets = set()
    for d, causal, n_max, emu, slots, group, persist, alg, bn in rows:
        key = (int(d), int(emu), int(slots), int(persist), int(alg), int(bn))
        assert key in compiled, f"table row {key} is not a compiled schedule"
        assert int(group) >= 1
        buckets.add((int(d), int(causal), n_max))
    for d in (64, 128):
        for causal in (0, 1):
            assert (d, causal, "INT64_MAX") in buckets, f"no open-ended bucket for d={d} causal={causal}"
    # and the pick for a few sizes agrees with the table row that covers it
    for d in (64, 128):
        for causal in (False, True):
            for N in (1000, 5000, 20000):
                sid, _ = fa.pick_schedule(N, d, causal)
                s = fa.schedules()[sid]
                row = next(r for r in rows if int(r[0]) == d and int(r[1]) == int(causal)
                           and (r[2] == "INT64_MAX" or N <= int(r[2])))
                assert (s["emu_every"], s["kv_slots"], s["persistent"], s["algorithm"], s["key_tile"]) == \
                    (int(row[3]), int(row[4]), int(row[6]), int(row[7]), int(row[8]))


def test_build_entry_does_not_need_the_library():
    # the build step must not import the package (its __init__ loads the library
    # the build step is about to create), so a fresh checkout can build
    import subprocess
    import sys
    import os
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    code = ("import sys, __graft_entry__ as g\n"
            "m = g._load_by_path('_b', 'attention_forward_17_b200/build.py')\n"
            "assert callable(m.build) and m.library_path().endswith('libfa_b200.so')\n"
            "assert 'attention_forward_17_b200' not in sys.modules, 'package imported'\n")
    r = subprocess.run([sys.executable, "-c", code], cwd=root, capture_output=True, text=True)
    assert r.returncode == 0, r.stderr
