"""The two-tile kernel's barrier protocol (TMA producer, MMA warp, softmax warps, epilogue),
checked on a CPU model under random interleavings (tests/handoff_model.py).

* The model's barrier follows the PTX parity rule, including the aliasing of a waiter two
  phases behind.
* Both MMA schedules of the kernel, P over S (d = 128, e4m3) and P in columns of its own
  (d = 64, bf16), finish every block, and every consumer sees the right block's data.
  That holds for TMA copies landing in any order, padding-only warps anywhere but warp 0,
  and several units of unequal, possibly empty, tiles per CTA.
* Leaving out any one wait is caught, as a wrong read, an overwrite in use or a deadlock.
  - Leaving out the padding-only warps' wait reproduces what a B200 showed for an earlier
    build: P.V ran on a P still holding an older block, while the row statistics (and so
    the LSE) stayed right.
  - Leaving out the ring-position rule of P over S's early first S deadlocks: K_0 of the
    next unit would wait for a ring slot this unit has not released yet.
"""
import random

import pytest

from tests import handoff_model as H

SEEDS = range(400)
SCHEDULES = {"separate P": True, "P over S": False}
ONLY_SEPARATE_P = {"s_free", "p_free", "idle_p_free"}
ONLY_P_OVER_S = {"ring_rule"}


def outcomes(separate_p, drop=()):
    races, deadlocks = [], []
    for seed in SEEDS:
        try:
            H.run_random(seed, separate_p=separate_p, drop=drop)
        except H.Race as e:
            races.append(str(e))
        except H.Deadlock as e:
            deadlocks.append(str(e))
    return races, deadlocks


def test_barrier_follows_the_parity_rule():
    b = H.Barrier("b", 2)
    # phase 0 in progress: waiting for parity 0 blocks, parity 1 (the phase "before") passes
    assert not b.done(0) and b.done(1)
    b.arrive()
    assert not b.done(0)
    b.arrive()  # phase 0 completes
    assert b.done(0) and not b.done(1)
    b.arrive()
    b.arrive()  # phase 1 completes: a waiter still on phase 0 now sees it as not done
    assert not b.done(0) and b.done(1)


def test_random_ctas_cover_the_kernel_geometry():
    seen = dict(empty_tile=False, unequal_tiles=False, units=False, idle=False, empty_unit=False)
    for seed in SEEDS:
        c = H.random_cta(random.Random(seed))
        seen["empty_tile"] |= any(0 in n and max(n) > 0 for n in c.units)
        seen["unequal_tiles"] |= any(n[0] != n[1] and min(n) > 0 for n in c.units)
        seen["units"] |= len(c.units) >= 4
        seen["idle"] |= any(any(s) for s in c.idle)
        seen["empty_unit"] |= any(max(n) == 0 for n in c.units)
    assert all(seen.values()), seen


@pytest.mark.parametrize("schedule", SCHEDULES)
def test_schedule_is_race_and_deadlock_free(schedule):
    races, deadlocks = outcomes(SCHEDULES[schedule])
    assert not races and not deadlocks, (races[:3], deadlocks[:3])


CASES = [(s, w) for s in SCHEDULES for w in H.Cta.WAITS
         if not (SCHEDULES[s] and w in ONLY_P_OVER_S)
         and not (not SCHEDULES[s] and w in ONLY_SEPARATE_P)]


@pytest.mark.parametrize("schedule,wait", CASES, ids=[f"{s}-{w}" for s, w in CASES])
def test_every_wait_is_needed(schedule, wait):
    races, deadlocks = outcomes(SCHEDULES[schedule], drop=(wait,))
    assert races or deadlocks, f"leaving out {wait} went unnoticed"


def test_idle_warp_race_reads_an_older_p():
    races, _ = outcomes(True, drop=("idle_p_free",))
    assert any(".V of" in r and "read warp" in r for r in races), races[:5]


def test_ring_rule_prevents_a_deadlock():
    races, deadlocks = outcomes(False, drop=("ring_rule",))
    assert deadlocks and not races, (races[:3], deadlocks[:3])
