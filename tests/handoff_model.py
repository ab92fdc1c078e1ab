"""A discrete-event model of the hand-offs between the MMA warp and the softmax warps of one
CTA of the two-tile forward kernel, for checking its barrier protocol on the CPU.

What it models, in the kernel's terms:

* mbarriers with an expected arrival count and a phase.  A parity wait succeeds once the
  phase of that parity has completed, i.e. while the current phase's parity differs from
  it (the PTX ``mbarrier.try_wait.parity`` rule).  Arrivals that spill into a later phase,
  and a waiter that falls two phases behind, are what this model exists to catch.
* the tensor pipe: MMAs and commits complete in issue order, each at a moment the scheduler
  picks; a commit arrives on its barrier once everything issued before it has completed.
* TMEM contents as (unit, block) tags: S_t written by an S MMA and read by the softmax
  warps; P_t written by each softmax warp (its 32 lanes) and read by P.V; O_t, which the
  softmax rescales between blocks.
* softmax warps, four per tile.  A warp whose 32 rows are all padding skips the loads and
  the math but keeps every hand-off (one arrival per warp stands for its 32 threads).
* two schedules: P written over S (the next S_t is issued after P_t.V), and P in columns
  of its own (the next block's S_t is issued once every warp has read S_t, before P_t.V).

Not modelled: TMA loads and the K/V ring, the Q buffers and the epilogue; they have
barriers of their own and the GPU tests cover them.

Test infrastructure only: nothing here is used by the library.
"""
import random


class Race(AssertionError):
    """A consumer saw data of the wrong block, or data was overwritten while in use."""


class Deadlock(AssertionError):
    """Nothing can run, but work remains."""


class Barrier:
    def __init__(self, name, count):
        self.name, self.count = name, count
        self.pending, self.phase = count, 0

    def arrive(self):
        self.pending -= 1
        if self.pending == 0:
            self.phase += 1
            self.pending = self.count

    def done(self, parity):
        """try_wait.parity: the phase with this parity has completed."""
        return (self.phase & 1) != parity


WARPS = 4
TILES = 2


class Cta:
    """units: per unit, the key blocks of each tile, e.g. [(3, 4), (0, 2)].
    idle: per unit, per tile, the set of warps whose rows are all padding.
    separate_p: P in columns of its own (else P over S).
    drop: waits to leave out, for planting a mistake: "s_free" (the MMA warp's wait before
    the next S), "p_free" (a softmax warp's wait before writing P and O), "idle_p_free" (a
    padding-only warp's wait before it arrives on p_full); separate P only."""

    WAITS = ("s_free", "p_free", "idle_p_free")

    def __init__(self, units, idle, separate_p=True, drop=()):
        assert set(drop) <= set(self.WAITS)
        self.units, self.idle = units, idle
        self.sep, self.drop = separate_p, set(drop)
        self.bars = {}
        for t in range(TILES):
            self.bars["s_full", t] = Barrier(f"s_full{t}", 1)
            self.bars["p_full", t] = Barrier(f"p_full{t}", WARPS)
            if separate_p:
                self.bars["s_free", t] = Barrier(f"s_free{t}", WARPS)
                self.bars["p_free", t] = Barrier(f"p_free{t}", 1)
        self.S = [None] * TILES
        self.P = [[None] * WARPS for _ in range(TILES)]
        self.s_unread = [set() for _ in range(TILES)]  # warps yet to load the current S_t
        self.pv_in_flight = [0] * TILES
        self.pipe = []
        self.pv_done = []

    # ---------------------------------------------------------------- tensor pipe
    def issue(self, op):
        if op[0] == "PV":
            self.pv_in_flight[op[1]] += 1
        self.pipe.append(op)

    def complete_one(self):
        op = self.pipe.pop(0)
        if op[0] == "S":
            _, t, tag = op
            if self.s_unread[t]:
                raise Race(f"S_{t} of {tag} written before warps {sorted(self.s_unread[t])} "
                           f"loaded S of {self.S[t]}")
            self.S[t] = tag
            self.s_unread[t] = set(range(WARPS)) - self.idle[tag[0]][t]
            if not self.sep:
                self.P[t] = [None] * WARPS  # P lives in S's columns
        elif op[0] == "PV":
            _, t, tag = op
            for w in range(WARPS):
                if w not in self.idle[tag[0]][t] and self.P[t][w] != tag:
                    raise Race(f"P_{t}.V of {tag} read warp {w}'s P of {self.P[t][w]}")
            self.pv_in_flight[t] -= 1
            self.pv_done.append((t, tag))
        else:
            self.bars[op[1]].arrive()

    # ---------------------------------------------------------------- MMA warp
    def _wait(self, key, parity):
        bar = self.bars[key]
        return lambda: bar.done(parity)

    def mma(self):
        pn = [0] * TILES  # p_full waits per tile
        sf = [0] * TILES  # s_free waits per tile (separate P)
        for u, n in enumerate(self.units):
            nblk = max(n)
            if nblk == 0:
                continue
            for t in range(TILES):
                if n[t]:
                    self.issue(("S", t, (u, 0)))
                    self.issue(("commit", ("s_full", t)))
            yield None
            for it in range(nblk):
                if self.sep and it + 1 < nblk:
                    for t in range(TILES):
                        if it + 1 >= n[t]:
                            continue
                        if "s_free" not in self.drop:
                            yield self._wait(("s_free", t), sf[t] & 1)
                        sf[t] += 1
                        self.issue(("S", t, (u, it + 1)))
                        self.issue(("commit", ("s_full", t)))
                for t in range(TILES):
                    if it >= n[t]:
                        continue
                    yield self._wait(("p_full", t), pn[t] & 1)
                    pn[t] += 1
                    self.issue(("PV", t, (u, it)))
                    if self.sep:
                        self.issue(("commit", ("p_free", t)))
                    elif it + 1 < n[t]:
                        self.issue(("S", t, (u, it + 1)))
                        self.issue(("commit", ("s_full", t)))
                yield None

    # ---------------------------------------------------------------- softmax warp
    def softmax(self, t, w):
        sn = 0  # S blocks of this tile so far
        for u, n in enumerate(self.units):
            nt = n[t]
            if nt == 0:
                continue
            idle = w in self.idle[u][t]
            for it in range(nt):
                yield self._wait(("s_full", t), sn & 1)
                sn += 1
                if not idle:
                    if self.S[t] != (u, it):
                        raise Race(f"softmax {t}.{w} loaded S of {self.S[t]} for {(u, it)}")
                    self.s_unread[t].discard(w)
                yield None
                if self.sep and it + 1 < nt:
                    self.bars["s_free", t].arrive()
                if idle:
                    if self.sep and "idle_p_free" not in self.drop and sn > 1:
                        yield self._wait(("p_free", t), sn & 1)
                    self.bars["p_full", t].arrive()
                    continue
                if self.sep and "p_free" not in self.drop and sn > 1:
                    yield self._wait(("p_free", t), sn & 1)
                # O rescale and P stores: the previous P.V must be complete
                if self.pv_in_flight[t]:
                    raise Race(f"softmax {t}.{w} wrote P/O of {(u, it)} while P.V in flight")
                self.P[t][w] = (u, it)
                yield None
                self.bars["p_full", t].arrive()

    # ---------------------------------------------------------------- scheduler
    def run(self, rng, max_steps=200000):
        """Interleave the actors at random (each with a random speed) until all finish."""
        actors = [self.mma()] + [self.softmax(t, w) for t in range(TILES) for w in range(WARPS)]
        speed = [rng.uniform(0.02, 1.0) for _ in range(len(actors) + 1)]  # last: the pipe
        cond = [None] * len(actors)
        live = list(range(len(actors)))
        for _ in range(max_steps):
            runnable = [i for i in live if cond[i] is None or cond[i]()]
            if self.pipe:
                runnable.append(len(actors))
            if not runnable:
                if live:
                    raise Deadlock(f"{len(live)} actors blocked, pipe empty")
                break
            i = rng.choices(runnable, weights=[speed[j] for j in runnable])[0]
            if i == len(actors):
                self.complete_one()
                continue
            try:
                cond[i] = next(actors[i])
            except StopIteration:
                live.remove(i)
        else:
            raise Deadlock("step limit")
        want = sorted((t, (u, it)) for u, n in enumerate(self.units)
                      for t in range(TILES) for it in range(n[t]))
        if sorted(self.pv_done) != want:
            raise Race("not every block's P.V completed")


def random_cta(rng, separate_p=True, drop=()):
    """One to four units per CTA, 0-4 key blocks per tile, random padding-only warps (warp 0
    of a tile with keys always holds a valid row)."""
    units, idle = [], []
    for _ in range(rng.randint(1, 4)):
        n = (rng.randint(0, 4), rng.randint(0, 4))
        units.append(n)
        idle.append([set(w for w in (1, 2, 3) if rng.random() < 0.5) for _ in range(TILES)])
    return Cta(units, idle, separate_p, drop)


def run_random(seed, **kw):
    rng = random.Random(seed)
    cta = random_cta(rng, **kw)
    cta.run(rng)
    return cta
