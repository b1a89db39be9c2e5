"""Model check of the attention kernels' K/V ring protocol, on the CPU.

The producer fills a ring of SLOTS shared-memory slots in a fixed order (per
query tile: K_0, K_1, K_2, then V_t followed by K_{t+3}); each load's slot is
reused SLOTS loads later.  A consumer waits for its load with an mbarrier
*parity* wait, which is only sound if the slot's previous load has already
completed when the wait starts; otherwise the wait can mistake that older
phase for its own and read a half-written tile.  So for every load i, the
consumer of load i must have observed (through its own earlier waits) the
completion of load i - SLOTS.

What each consumer has observed before it waits, per kernel:
  score issuer, S(m), one-tile-per-CTA kernel: every K_{m'<m} (it consumed
      them) and every V_{t<=m-3} (it waited for the product of step m-3);
  score issuer, S(m), split-KV ping-pong kernel: every K_{m'<m} only (it waits
      for the softmax to have read S(m-2), not for any product);
  output issuer, O += P_t V_t (both kernels): every K_{m<=t} (it waited for
      P_t, which needed S(t), which needed K_t and the K tiles before it) and
      every V_{t'<t} (it consumed them).
Persistent launches run several tiles through one ring with global step and
load counts, so sequences of tiles are checked too (for the launch forms that
do that; the ping-pong kernel would not be sound across tiles and runs one
tile per CTA).

This is the reasoning that found a real race (the output issuer used to wait
for V_t before P_t); the last tests check that the model flags that order and
a three-slot ring.

The two-query-tile kernel (algorithm 2) loads K_0, V_0, K_1, V_1, ... once for
both of its query tiles, and each of its two issuers visits every load in that
order: it waits for the load to land and then uses it (products, then a
release by commit) or, for key tiles its query tile does not need under the
causal mask, releases it by a plain arrival.  Each release needs both issuers.
Two things must hold: a parity wait on load i starts after the waiter observed
load i - SLOTS (true when every visit waits, in order), and a release arrival
for load i lands in load i's phase of the slot's empty barrier, which holds
once load i has landed (the producer issued it after load i - SLOTS was
released by both issuers).  The model below checks both for every compiled
depth and every pair of key-tile counts, and flags an issuer that releases
unused loads without waiting for them.
"""
import random

import pytest

import attention_forward_17_b200 as fa


def tile_loads(n):
    """Load order of one query tile with n key tiles: (kind, key tile index)."""
    seq = [("K", m) for m in range(min(3, n))]
    for t in range(n):
        seq.append(("V", t))
        if t + 3 < n:
            seq.append(("K", t + 3))
    return seq


def loads_for(tiles):
    """Global load sequence over several query tiles; steps counted globally."""
    seq, base = [], 0
    for n in tiles:
        seq += [(k, base + x) for k, x in tile_loads(n)]
        base += n
    return seq


def observed(kind, step, pred_kind, pred_step, algorithm, v_before_p=False):
    if kind == "K":                      # score issuer at S(step)
        if pred_kind == "K":
            return pred_step < step
        return algorithm == 0 and pred_step <= step - 3
    # output issuer at step: after P_step (or, in the faulty order, before it)
    k_seen = step - 1 if v_before_p else step
    return (pred_kind == "K" and pred_step <= k_seen) or (pred_kind == "V" and pred_step < step)


def violations(tiles, slots, algorithm, v_before_p=False):
    seq = loads_for(tiles)
    bad = 0
    for i, (kind, step) in enumerate(seq):
        j = i - slots
        if j >= 0 and not observed(kind, step, *seq[j], algorithm, v_before_p):
            bad += 1
    return bad


def compiled_rings():
    """Rings of the one-tile kernels (algorithms 0 and 1); the two-tile kernel's
    ring is modelled below."""
    return sorted({(s["kv_slots"], s["algorithm"]) for s in fa.schedules() if s["algorithm"] < 2})


def compiled_multi_tile_rings():
    """Rings that continue across query tiles (the persistent launch forms)."""
    return sorted({(s["kv_slots"], s["algorithm"]) for s in fa.schedules() if s["persistent"]})


@pytest.mark.parametrize("slots,algorithm", compiled_rings())
def test_every_compiled_ring_is_sound_for_one_tile(slots, algorithm):
    for n in range(1, 70):
        assert violations([n], slots, algorithm) == 0, f"n={n}"


@pytest.mark.parametrize("slots,algorithm", compiled_multi_tile_rings())
def test_every_compiled_ring_is_sound_across_tiles(slots, algorithm):
    rng = random.Random(slots * 10 + algorithm)
    for _ in range(2000):
        tiles = [rng.randint(1, 20) for _ in range(rng.randint(1, 6))]
        assert violations(tiles, slots, algorithm) == 0, f"tiles={tiles}"


def test_model_flags_the_old_wait_order():
    # waiting for V_t before P_t was racy at the old default depth of five
    assert sum(violations([n], 5, 0, v_before_p=True) for n in range(1, 40)) > 0


def test_model_flags_a_three_slot_ring():
    assert sum(violations([n], 3, 0) for n in range(1, 40)) > 0
    assert sum(violations([n], 3, 1) for n in range(1, 40)) > 0


def test_ping_pong_kernel_is_never_persistent():
    # across a tile boundary the ping-pong score issuer could reach a K tile whose
    # slot predecessor is a V tile of the previous query tile, which it never
    # observes: the model flags it, so that kernel runs one tile per CTA only
    rng = random.Random(7)
    assert any(violations([rng.randint(1, 20) for _ in range(4)], 4, 1) for _ in range(200))
    assert not any(s["persistent"] for s in fa.schedules() if s["algorithm"] == 1)


def test_model_flags_an_odd_ring_for_the_ping_pong_kernel():
    # with P in shared memory the score issuer observes no V load, so a K tile's
    # slot predecessor must itself be a K tile: odd depths break that
    assert sum(violations([n], 5, 1) for n in range(1, 40)) > 0
    assert all(s["kv_slots"] % 2 == 0 for s in fa.schedules() if s["algorithm"] == 1)


# ------------------------------------------------------------------ two-query-tile kernel
def two_tile_issuer_events(n0, n1, ahead=1, release_k_early=False, more=()):
    """The ring events of the multi-tile kernel's MMA issuer, in program
    order, for key-tile counts n0 (tile 0), n1 (tile 1) and `more` (further
    tiles of a CTA that holds three): ("wait", L),
    ("use", L), ("release", L) with L the load index (K_j = 2j, V_j = 2j+1).
    `ahead` is how many score products run ahead of the softmax (1 with one
    score buffer per tile, 2 with two).  release_k_early models a faulty
    variant that releases the next K tile right after tile 0's score product."""
    ev, waited = [], [-1]

    def wait(ld):                       # waits for every load up to ld, in order
        while waited[0] < ld:
            waited[0] += 1
            ev.append(("wait", waited[0]))

    counts = (n0, n1) + tuple(more)
    n_kv = max(counts)
    for j in range(min(ahead, n_kv)):
        wait(2 * j)
        for n_i in counts:
            if j < n_i:
                ev.append(("use", 2 * j))
        ev.append(("release", 2 * j))
    for j in range(n_kv):
        for ti, n_i in enumerate(counts):
            if j >= n_i:
                continue
            wait(2 * j + 1)
            ev.append(("use", 2 * j + 1))
            if j + ahead < n_i:
                wait(2 * (j + ahead))
                ev.append(("use", 2 * (j + ahead)))
                if release_k_early and ti == 0:
                    ev.append(("release", 2 * (j + ahead)))
        ev.append(("release", 2 * j + 1))
        if j + ahead < n_kv and not (release_k_early and j + ahead < n0):
            ev.append(("release", 2 * (j + ahead)))
    return ev, 2 * n_kv


def two_tile_violations(n0, n1, slots, **kw):
    """Unsound parity waits, uses of unobserved or released loads, and loads
    released twice or never, for the issuer's event sequence."""
    ev, loads = two_tile_issuer_events(n0, n1, **kw)
    bad = 0
    landed, released = set(), set()
    for kind, ld in ev:
        if kind == "wait":
            # a parity wait on load ld is sound once the slot's previous load was observed
            if ld >= slots and (ld - slots) not in landed:
                bad += 1
            # and the producer issues load ld only after load ld - slots was released:
            # a release that comes later in the issuer's own order is a deadlock
            if ld >= slots and (ld - slots) not in released:
                bad += 1
            landed.add(ld)
        elif kind == "use":
            if ld not in landed or ld in released:
                bad += 1
        else:
            if ld not in landed or ld in released:
                bad += 1
            released.add(ld)
    # the producer reuses a slot after the release of its previous load: every load must be released
    bad += loads - len(released)
    return bad


def compiled_two_tile_rings():
    """(depth, score products ahead, query tiles per CTA) of every compiled
    multi-tile schedule."""
    return sorted({(s["kv_slots"], 2 if (s["algorithm"] - 2) & 1 else 1, 3 if (s["algorithm"] - 2) & 8 else 2)
                   for s in fa.schedules() if s["algorithm"] >= 2})


@pytest.mark.parametrize("slots,ahead,nt", compiled_two_tile_rings())
def test_two_tile_ring_is_sound(slots, ahead, nt):
    for n in range(0, 40):
        if nt == 2:
            # non-causal (equal counts), causal (tile 0 one to three key tiles short,
            # for key tiles of 192, 128 and 64 rows), and a second tile past the end
            # of the sequence (no keys)
            for n0 in {n, n - 1, n - 2}:
                if n0 >= 1:
                    assert two_tile_violations(n0, n, slots, ahead=ahead) == 0, (n0, n)
            assert two_tile_violations(n + 1, 0, slots, ahead=ahead) == 0
        else:
            # three tiles: equal counts, causal steps of one or two key tiles per
            # query tile, and the last one or two tiles past the end
            for step in (0, 1, 2):
                if n - 2 * step >= 1:
                    assert two_tile_violations(n - 2 * step, n - step, slots, ahead=ahead, more=(n,)) == 0
            assert two_tile_violations(n + 1, n + 1, slots, ahead=ahead, more=(0,)) == 0
            assert two_tile_violations(n + 1, 0, slots, ahead=ahead, more=(0,)) == 0


def test_three_tile_schedules_exist():
    assert any((s["algorithm"] - 2) & 8 for s in fa.schedules() if s["algorithm"] >= 2)


def test_model_flags_a_shallow_ring_with_two_score_buffers():
    # K_{j+2} is needed while V_j is still unreleased: three slots deadlock
    assert sum(two_tile_violations(n, n, 3, ahead=2) for n in range(3, 20)) > 0
    assert all(s["kv_slots"] >= 4 for s in fa.schedules() if s["algorithm"] >= 2 and (s["algorithm"] - 2) & 1)


def test_model_flags_an_early_key_release():
    for ahead in (1, 2):
        assert sum(two_tile_violations(n, n, 5, ahead=ahead, release_k_early=True)
                   for n in range(3, 20)) > 0


# ------------------------------------------------------------------ P barriers of the two-tile kernel
def p_barrier_unsound_waits(n, ahead, nbufs):
    """Parity waits of the issuer on the P barriers that the softmax can have
    run two phases past.  The softmax is modelled as fast as its inputs allow:
    it releases P(k) as soon as S(k) exists, and S(k) is issued in the prologue
    (k < ahead) or right after the issuer consumed P(k - ahead).  P(k) lives on
    barrier k % nbufs (phase k // nbufs).  When the issuer waits for P(j) it has
    consumed P(0..j-1), so the softmax can have released P(0 .. j-1+ahead); the
    wait is unsound if that includes the next phase of the same barrier, P(j+nbufs)."""
    bad = 0
    for j in range(n):
        released_up_to = min(n - 1, j - 1 + ahead)
        if j + nbufs <= released_up_to:
            bad += 1
    return bad


def test_p_barriers_cannot_run_two_phases_ahead():
    for s in fa.schedules():
        if s["algorithm"] < 2:
            continue
        ahead = nbufs = 2 if (s["algorithm"] - 2) & 1 else 1
        for n in range(1, 40):
            assert p_barrier_unsound_waits(n, ahead, nbufs) == 0, (s, n)


def test_model_flags_one_p_barrier_with_two_score_buffers():
    # the first version of the double-buffered kernel kept one P barrier per tile:
    # its issuer's waits ran out of time once the softmax got a step ahead
    assert sum(p_barrier_unsound_waits(n, 2, 1) for n in range(3, 20)) > 0
