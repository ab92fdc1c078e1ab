"""The forward kernel's barrier protocol (TMA producer, MMA warp, softmax warps, epilogue),
checked on a CPU model under random interleavings (tests/handoff_model.py).

* The model's barrier follows the PTX parity rule, including the aliasing of a waiter two
  phases behind.
* The kernel's three configurations finish every block, and every consumer sees the right
  block's data:
  - two tiles with P over S (d = 128, e4m3);
  - two tiles with P in columns of its own (d = 64, bf16);
  - one tile with P over S (decode and short query axes).
  That holds for TMA copies landing in any order, padding-only warps anywhere but warp 0,
  and several units of unequal, possibly empty, tiles per CTA.
* Leaving out any one wait is caught, as a wrong read, an overwrite in use or a deadlock.
  - Leaving out the padding-only warps' wait reproduces what a B200 showed for an earlier
    build: P.V ran on a P still holding an older block, while the row statistics (and so
    the LSE) stayed right.
  - Leaving out the ring-position rule of P over S's early first S deadlocks: K_0 of the
    next unit would wait for a ring slot this unit has not released yet.
* A design under study, one MMA-issuing warp per tile with P over S, is checked the same
  way before any kernel code: each issuer must walk every ring entry in order, also those
  its tile does not read, before it releases them (both issuers release every entry).
* With one tile, two waits are implied by others, and the model shows it:
  - the ring-position rule always holds: the tile ends on its unit's last block;
  - the MMA warp's wait for the released O: the next unit's first P.V already waits for
    every warp's P, which each warp writes only after reading the last O out.
"""
import random

import pytest

from tests import handoff_model as H

SEEDS = range(400)
SCHEDULES = {
    "two tiles, separate P": dict(separate_p=True, tiles=2),
    "two tiles, P over S": dict(separate_p=False, tiles=2),
    "one tile, P over S": dict(separate_p=False, tiles=1),
    # a design under study: one MMA-issuing warp per tile
    "two tiles, P over S, two issuers": dict(separate_p=False, tiles=2, two_issuers=True),
}
ONLY_SEPARATE_P = {"s_free", "p_free", "idle_p_free"}
ONLY_TWO_ISSUERS = {"every_index"}
IMPLIED_WITH_ONE_TILE = {"ring_rule", "o_empty"}


def outcomes(schedule, drop=()):
    races, deadlocks = [], []
    for seed in SEEDS:
        try:
            H.run_random(seed, drop=drop, **SCHEDULES[schedule])
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
        c = H.random_cta(random.Random(seed), tiles=2)
        seen["empty_tile"] |= any(0 in n and max(n) > 0 for n in c.units)
        seen["unequal_tiles"] |= any(n[0] != n[1] and min(n) > 0 for n in c.units)
        seen["units"] |= len(c.units) >= 4
        seen["idle"] |= any(any(s) for s in c.idle)
        seen["empty_unit"] |= any(max(n) == 0 for n in c.units)
    assert all(seen.values()), seen


@pytest.mark.parametrize("schedule", SCHEDULES)
def test_schedule_is_race_and_deadlock_free(schedule):
    races, deadlocks = outcomes(schedule)
    assert not races and not deadlocks, (races[:3], deadlocks[:3])


def applies(schedule, wait):
    kw = SCHEDULES[schedule]
    if wait in ONLY_SEPARATE_P:
        return kw["separate_p"]
    if wait in ONLY_TWO_ISSUERS:
        return kw.get("two_issuers", False)
    if wait == "ring_rule" and kw["separate_p"]:
        return False  # the separate-P schedule has no early first S
    return not (kw["tiles"] == 1 and wait in IMPLIED_WITH_ONE_TILE)


CASES = [(s, w) for s in SCHEDULES for w in H.Cta.WAITS if applies(s, w)]


@pytest.mark.parametrize("schedule,wait", CASES, ids=[f"{s}-{w}" for s, w in CASES])
def test_every_wait_is_needed(schedule, wait):
    races, deadlocks = outcomes(schedule, drop=(wait,))
    assert races or deadlocks, f"leaving out {wait} went unnoticed"


@pytest.mark.parametrize("wait", sorted(IMPLIED_WITH_ONE_TILE))
def test_waits_implied_with_one_tile(wait):
    races, deadlocks = outcomes("one tile, P over S", drop=(wait,))
    assert not races and not deadlocks, (races[:3], deadlocks[:3])


def test_idle_warp_race_reads_an_older_p():
    races, _ = outcomes("two tiles, separate P", drop=("idle_p_free",))
    assert any(".V of" in r and "read warp" in r for r in races), races[:5]


def test_ring_rule_prevents_a_deadlock():
    races, deadlocks = outcomes("two tiles, P over S", drop=("ring_rule",))
    assert deadlocks and not races, (races[:3], deadlocks[:3])
