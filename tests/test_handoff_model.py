"""The two-tile kernel's MMA / softmax hand-off protocol, checked on a CPU model under random
interleavings (tests/handoff_model.py).

* The model's barrier follows the PTX parity rule, including the aliasing of a waiter two
  phases behind.
* Both schedules of the kernel, P over S (d = 128, e4m3) and P in columns of its own
  (d = 64 bf16), finish every block with every consumer seeing the right block's data,
  with padding-only warps anywhere but warp 0 and units of unequal, possibly empty, tiles.
* Leaving out any one wait of the separate-P schedule is caught.  Leaving out the
  padding-only warps' wait reproduces what a B200 showed for an earlier build: P.V ran on
  a P still holding an older block, while the statistics (and so the LSE) stayed right.
"""
import pytest

from tests import handoff_model as H

SEEDS = range(400)


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


@pytest.mark.parametrize("separate_p", [True, False], ids=["separate P", "P over S"])
def test_schedule_is_race_free(separate_p):
    for seed in SEEDS:
        H.run_random(seed, separate_p=separate_p)


def test_model_covers_the_kernel_geometry():
    # the random CTAs include empty tiles, unequal tiles, several units and idle warps
    seen = dict(empty=False, unequal=False, units=False, idle=False)
    import random
    for seed in SEEDS:
        c = H.random_cta(random.Random(seed))
        seen["empty"] |= any(0 in n and max(n) > 0 for n in c.units)
        seen["unequal"] |= any(n[0] != n[1] and min(n) > 0 for n in c.units)
        seen["units"] |= len(c.units) >= 3
        seen["idle"] |= any(any(s) for s in c.idle)
    assert all(seen.values()), seen


@pytest.mark.parametrize("wait", H.Cta.WAITS)
def test_every_wait_of_the_separate_p_schedule_is_needed(wait):
    failures = 0
    for seed in SEEDS:
        try:
            H.run_random(seed, drop=(wait,))
        except (H.Race, H.Deadlock):
            failures += 1
    assert failures > 0, f"leaving out {wait} went unnoticed"


def test_idle_warp_race_reads_an_older_p():
    symptoms = []
    for seed in SEEDS:
        try:
            H.run_random(seed, drop=("idle_p_free",))
        except H.Race as e:
            symptoms.append(str(e))
    assert any(".V of" in s and "read warp" in s for s in symptoms), symptoms[:5]
