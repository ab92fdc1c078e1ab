"""A discrete-event model of one CTA of the forward kernel, for checking its barrier protocol
on the CPU: the TMA producer, the MMA warp, four softmax warps per tile and the epilogue,
with the hand-offs between them.  Two tiles per CTA (prefill) or one (decode and short
query axes, where the softmax warps write their own output and release O).

What it models, in the kernel's terms:

* mbarriers with an expected arrival count and a phase.  A parity wait succeeds once the
  phase of that parity has completed, i.e. while the current phase's parity differs from
  it (the PTX ``mbarrier.try_wait.parity`` rule).  Arrivals that spill into a later phase,
  and a waiter that falls two phases behind, are what this model exists to catch.
* TMA loads land in any order, each at a moment the scheduler picks, and arrive on their
  full barrier.  Q_t has a buffer per tile; K and V blocks share a ring of slots, loaded in
  the order Q_0, K_0, Q_1, V_0, K_1, V_1, ... per unit.
* the tensor pipe: MMAs and commits complete in issue order, each at a moment the scheduler
  picks; a commit arrives on its barrier once everything issued before it has completed.
  An MMA reads its shared-memory operands until it completes.
* TMEM contents as (unit, block) tags: S_t written by an S MMA and loaded by the softmax
  warps; P_t written by each softmax warp (its 32 lanes) and read by P.V; O_t accumulated
  by P.V, rescaled by the softmax between blocks and read out by the epilogue.
* softmax warps, four per tile.  A warp whose 32 rows are all padding skips the loads and
  the math but keeps every hand-off (one arrival per warp stands for its 32 threads; the
  epilogue's arrival stands for its warpgroup's).
* the two MMA schedules of the kernel:
  - P over S (d = 128 and e4m3): per block, P_t.V then the next S_t, tile by tile; a tile
    that finishes its unit issues the next unit's first S_t at once, when the ring entry
    that K_0 of that unit replaces was released by an earlier iteration (the ring-position
    rule);
  - P in columns of its own (d = 64, bf16): per block, the next S_t of every tile once its
    softmax has loaded S_t ("S read"), then P_t.V of every tile, each committed to
    "P.V done".

Not modelled: the row statistics the softmax posts for the epilogue, and the arithmetic.

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


class Cta:
    """units: per unit of this CTA, the key blocks of each tile, e.g. [(3, 4), (0, 2)].
    idle: per unit, per tile, the set of warps whose rows are all padding.
    separate_p: P in columns of its own (else P over S; the kernel uses separate P with two
    bf16 tiles at d = 64 only).
    slots: K/V ring slots (the kernel has 4 at d = 128 and 8 at d = 64 with two tiles, 2 and
    5 with one).
    tiles: 2, with an epilogue warpgroup; or 1, whose softmax warps write the output.
    drop: waits to leave out, for planting a mistake:
      "s_free"      the MMA warp's wait for "S read" before the next S (separate P);
      "p_free"      a softmax warp's wait for the previous P.V before writing P and O
                    (separate P);
      "idle_p_free" a padding-only warp's wait for the previous P.V before it arrives on
                    "P ready" (separate P);
      "ring_rule"   the ring-position condition on the early first S (P over S);
      "o_empty"     the MMA warp's wait for the epilogue before a unit's first P.V;
      "kv_empty"    the producer's wait for a free ring slot;
      "q_empty"     the producer's wait before it reloads a Q buffer;
      "every_index" (two issuers) an issuer's wait for a ring entry its tile does not read,
                    before it releases that entry.
    two_issuers: P over S with one MMA-issuing warp per tile (a design under study, not the
    kernel's): each walks every ring entry in order and releases each (kv_empty counts
    both), and a tile's early first S follows the same ring-position rule."""

    WAITS = ("s_free", "p_free", "idle_p_free", "ring_rule", "o_empty", "kv_empty", "q_empty",
             "every_index")

    def __init__(self, units, idle, separate_p=True, slots=None, drop=(), tiles=2,
                 two_issuers=False):
        assert set(drop) <= set(self.WAITS) and tiles in (1, 2)
        assert all(len(n) == tiles for n in units)
        assert not (two_issuers and (separate_p or tiles != 2))
        self.units, self.idle = units, idle
        self.sep, self.drop, self.nt = separate_p, set(drop), tiles
        self.two_issuers = two_issuers
        self.slots = slots or ((8 if separate_p else 4) if tiles == 2 else 2)
        B = Barrier
        self.bars = {}
        for s in range(self.slots):
            self.bars["kv_full", s] = B(f"kv_full{s}", 1)
            self.bars["kv_empty", s] = B(f"kv_empty{s}", 2 if two_issuers else 1)
        o_empty_count = 1 if tiles == 2 else WARPS  # the epilogue, or every softmax warp
        for t in range(tiles):
            for name, count in (("q_full", 1), ("q_empty", 1), ("s_full", 1),
                                ("p_full", WARPS), ("o_full", 1), ("o_empty", o_empty_count),
                                ("s_free", WARPS), ("p_free", 1)):
                self.bars[name, t] = B(f"{name}{t}", count)
        self.kv = [None] * self.slots          # ring slot contents
        self.kv_readers = [0] * self.slots     # MMAs in flight reading the slot
        self.q = [None] * self.nt
        self.q_readers = [0] * self.nt
        self.S = [None] * self.nt
        self.P = [[None] * WARPS for _ in range(self.nt)]
        self.s_unread = [set() for _ in range(self.nt)]  # warps yet to load the current S_t
        self.O = [None] * self.nt                # (unit, blocks accumulated)
        self.o_read = [True] * self.nt           # the epilogue has read the last unit's O_t
        self.pv_in_flight = [0] * self.nt
        self.pipe = []                         # tensor pipe, in issue order
        self.issued, self.n_done = 0, 0        # MMAs issued / completed
        self.last_op = {}                      # per issuer: number of its latest MMA
        self.commits = []                      # (MMA number to wait for, barrier)
        self.tma = []                          # loads in flight, any completion order
        self.pv_done = []
        self.epilogue_done = []
        self.o_readers = 0                     # readers of the current O done (one tile)

    # ---------------------------------------------------------------- async engines
    def issue(self, op, who=0):
        if op[0] == "S":
            self.kv_readers[op[2]] += 1
            self.q_readers[op[1]] += 1
        else:
            self.kv_readers[op[2]] += 1
            self.pv_in_flight[op[1]] += 1
        self.pipe.append(op)
        self.issued += 1
        self.last_op[who] = self.issued  # MMA number k has completed once k <= n_done

    def commit(self, key, who=0):
        """tcgen05.commit: arrive on the barrier once every MMA this issuer has issued so far
        has completed (another issuer's MMAs do not count)."""
        self.commits.append((self.last_op.get(who, 0), key))

    def fire_commit(self, i):
        self.bars[self.commits.pop(i)[1]].arrive()

    def ready_commits(self):
        return [i for i, (k, _) in enumerate(self.commits) if k <= self.n_done]

    def complete_mma(self):
        op = self.pipe.pop(0)
        self.n_done += 1
        if op[0] == "S":
            _, t, slot, (u, it) = op
            if self.kv[slot] != ("K", u, it) or self.q[t] != u:
                raise Race(f"S_{t} of {(u, it)} read K {self.kv[slot]} and Q of unit {self.q[t]}")
            self.kv_readers[slot] -= 1
            self.q_readers[t] -= 1
            if self.s_unread[t]:
                raise Race(f"S_{t} of {(u, it)} written before warps {sorted(self.s_unread[t])} "
                           f"loaded S of {self.S[t]}")
            self.S[t] = (u, it)
            self.s_unread[t] = set(range(WARPS)) - self.idle[u][t]
            if not self.sep:
                self.P[t] = [None] * WARPS  # P lives in S's columns
        elif op[0] == "PV":
            _, t, slot, (u, it) = op
            if self.kv[slot] != ("V", u, it):
                raise Race(f"P_{t}.V of {(u, it)} read V {self.kv[slot]}")
            for w in range(WARPS):
                if w not in self.idle[u][t] and self.P[t][w] != (u, it):
                    raise Race(f"P_{t}.V of {(u, it)} read warp {w}'s P of {self.P[t][w]}")
            if it == 0:
                if not self.o_read[t]:
                    raise Race(f"P_{t}.V of {(u, it)} overwrote O of {self.O[t]} before the epilogue read it")
                self.o_read[t] = False
            elif self.O[t] != (u, it):
                raise Race(f"P_{t}.V of {(u, it)} accumulated onto O of {self.O[t]}")
            self.O[t] = (u, it + 1)
            self.kv_readers[slot] -= 1
            self.pv_in_flight[t] -= 1
            self.pv_done.append((t, (u, it)))

    def complete_tma(self, i):
        kind, where, tag = self.tma.pop(i)
        if kind == "Q":
            if self.q_readers[where]:
                raise Race(f"Q_{where} of unit {tag} landed while an S MMA read the buffer")
            self.q[where] = tag
            self.bars["q_full", where].arrive()
        else:
            if self.kv_readers[where]:
                raise Race(f"{kind} of {tag} landed in slot {where} while an MMA read it")
            self.kv[where] = (kind,) + tag
            self.bars["kv_full", where].arrive()

    def _wait(self, key, parity):
        bar = self.bars[key]
        return lambda: bar.done(parity)

    # ---------------------------------------------------------------- TMA producer
    def producer(self):
        ld, qn = 0, [0] * self.nt

        def load_q(u, n, t):
            if n[t] == 0:
                return
            if qn[t] > 0 and "q_empty" not in self.drop:
                yield self._wait(("q_empty", t), (qn[t] - 1) & 1)
            self.tma.append(("Q", t, u))
            qn[t] += 1

        for u, n in enumerate(self.units):
            yield from load_q(u, n, 0)
            for it in range(max(n)):
                for kind in ("K", "V"):
                    slot = ld % self.slots
                    if ld >= self.slots and "kv_empty" not in self.drop:
                        yield self._wait(("kv_empty", slot), ((ld // self.slots) - 1) & 1)
                    self.tma.append((kind, slot, (u, it)))
                    ld += 1
                    if it == 0 and kind == "K":
                        for t in range(1, self.nt):
                            yield from load_q(u, n, t)
                yield None

    # ---------------------------------------------------------------- MMA warp
    def mma(self):
        st = dict(ld=0, qn=[0] * self.nt, pn=[0] * self.nt, on=[0] * self.nt, sf=[0] * self.nt)
        yield from (self._mma_separate_p(st) if self.sep else self._mma_p_over_s(st))

    def _wait_kv(self, st, index):
        return self._wait(("kv_full", index % self.slots), (index // self.slots) & 1)

    def _issue_s(self, st, t, slot, tag, n_t, who=0):
        """Q_t must have landed; then S_t, its commit, and Q_t's release after the last S_t."""
        yield self._wait(("q_full", t), st["qn"][t] & 1) if tag[1] == 0 else None
        if tag[1] == 0:
            st["qn"][t] += 1
        self.issue(("S", t, slot, tag), who)
        self.commit(("s_full", t), who)
        if tag[1] + 1 == n_t:
            self.commit(("q_empty", t), who)

    def _issue_pv(self, st, t, slot, tag, who=0):
        yield self._wait(("p_full", t), st["pn"][t] & 1)
        st["pn"][t] += 1
        if tag[1] == 0 and st["on"][t] > 0 and "o_empty" not in self.drop:
            yield self._wait(("o_empty", t), (st["on"][t] - 1) & 1)
        self.issue(("PV", t, slot, tag), who)

    def _mma_p_over_s(self, st):
        early = [False] * self.nt
        for ui, n in enumerate(self.units):
            n_next = self.units[ui + 1] if ui + 1 < len(self.units) else (0,) * self.nt
            early_next = [False] * self.nt
            nblk = max(n)
            if nblk == 0:
                continue
            ld_unit = st["ld"]
            slot_k = st["ld"] % self.slots
            yield self._wait_kv(st, st["ld"])
            st["ld"] += 1
            for t in range(self.nt):
                if n[t] and not early[t]:
                    yield from self._issue_s(st, t, slot_k, (ui, 0), n[t])
            self.commit(("kv_empty", slot_k))
            for it in range(nblk):
                slot_v = st["ld"] % self.slots
                yield self._wait_kv(st, st["ld"])
                st["ld"] += 1
                nxt = it + 1 < nblk
                ld_n = st["ld"]
                slot_n = ld_n % self.slots
                k_ready = False
                if nxt:
                    st["ld"] += 1
                for t in range(self.nt):
                    if it >= n[t]:
                        continue
                    yield from self._issue_pv(st, t, slot_v, (ui, it))
                    if it + 1 < n[t]:
                        if not k_ready:
                            yield self._wait_kv(st, ld_n)
                            k_ready = True
                        yield from self._issue_s(st, t, slot_n, (ui, it + 1), n[t])
                    else:
                        self.commit(("o_full", t))
                        st["on"][t] += 1
                        rule = 2 * (nblk - it) <= self.slots or "ring_rule" in self.drop
                        if n_next[t] > 0 and rule:
                            kq = ld_unit + 2 * nblk
                            yield self._wait_kv(st, kq)
                            yield from self._issue_s(st, t, kq % self.slots, (ui + 1, 0), n_next[t])
                            early_next[t] = True
                    yield None
                self.commit(("kv_empty", slot_v))
                if nxt:
                    self.commit(("kv_empty", slot_n))
            early = early_next

    def _mma_one_tile(self, t):
        """Two issuers: this warp issues tile t's MMAs only."""
        who = 1 + t
        st = dict(ld=0, qn=[0] * self.nt, pn=[0] * self.nt, on=[0] * self.nt)
        early = False
        for ui, n in enumerate(self.units):
            n_next = self.units[ui + 1] if ui + 1 < len(self.units) else (0,) * self.nt
            early_next = False
            nblk = max(n)
            if nblk == 0:
                continue
            ld_unit = st["ld"]
            slot_k = st["ld"] % self.slots
            yield self._wait_kv(st, st["ld"])
            st["ld"] += 1
            if n[t] and not early:
                yield from self._issue_s(st, t, slot_k, (ui, 0), n[t], who)
            self.commit(("kv_empty", slot_k), who)
            for it in range(nblk):
                slot_v = st["ld"] % self.slots
                yield self._wait_kv(st, st["ld"])
                st["ld"] += 1
                nxt = it + 1 < nblk
                ld_n = st["ld"]
                slot_n = ld_n % self.slots
                k_ready = False
                if nxt:
                    st["ld"] += 1
                if it < n[t]:
                    yield from self._issue_pv(st, t, slot_v, (ui, it), who)
                    if it + 1 < n[t]:
                        yield self._wait_kv(st, ld_n)
                        k_ready = True
                        yield from self._issue_s(st, t, slot_n, (ui, it + 1), n[t], who)
                    else:
                        self.commit(("o_full", t), who)
                        st["on"][t] += 1
                        rule = 2 * (nblk - it) <= self.slots or "ring_rule" in self.drop
                        if n_next[t] > 0 and rule:
                            kq = ld_unit + 2 * nblk
                            yield self._wait_kv(st, kq)
                            yield from self._issue_s(st, t, kq % self.slots, (ui + 1, 0),
                                                     n_next[t], who)
                            early_next = True
                yield None
                self.commit(("kv_empty", slot_v), who)
                if nxt:
                    # release K of the next block too, after waiting for it even when this
                    # tile does not read it: the entry's phase must be the current one
                    if not k_ready and "every_index" not in self.drop:
                        yield self._wait_kv(st, ld_n)
                    self.commit(("kv_empty", slot_n), who)
            early = early_next

    def _mma_separate_p(self, st):
        for ui, n in enumerate(self.units):
            nblk = max(n)
            if nblk == 0:
                continue
            slot_k = st["ld"] % self.slots
            yield self._wait_kv(st, st["ld"])
            st["ld"] += 1
            for t in range(self.nt):
                if n[t]:
                    yield from self._issue_s(st, t, slot_k, (ui, 0), n[t])
            self.commit(("kv_empty", slot_k))
            for it in range(nblk):
                slot_v = st["ld"] % self.slots
                yield self._wait_kv(st, st["ld"])
                st["ld"] += 1
                if it + 1 < nblk:
                    slot_n = st["ld"] % self.slots
                    yield self._wait_kv(st, st["ld"])
                    st["ld"] += 1
                    for t in range(self.nt):
                        if it + 1 >= n[t]:
                            continue
                        if "s_free" not in self.drop:
                            yield self._wait(("s_free", t), st["sf"][t] & 1)
                        st["sf"][t] += 1
                        yield from self._issue_s(st, t, slot_n, (ui, it + 1), n[t])
                    self.commit(("kv_empty", slot_n))
                for t in range(self.nt):
                    if it >= n[t]:
                        continue
                    yield from self._issue_pv(st, t, slot_v, (ui, it))
                    self.commit(("p_free", t))
                    if it + 1 == n[t]:
                        self.commit(("o_full", t))
                        st["on"][t] += 1
                self.commit(("kv_empty", slot_v))
                yield None

    # ---------------------------------------------------------------- softmax warp
    def softmax(self, t, w):
        sn = 0  # S blocks of this tile so far
        so = 0  # outputs of this tile written (one tile per CTA)
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
                # P stores, and (past the first block) the O rescale: the previous P.V must
                # be complete
                if self.pv_in_flight[t]:
                    raise Race(f"softmax {t}.{w} wrote P of {(u, it)} while P.V was in flight")
                if it > 0 and self.O[t] != (u, it):
                    raise Race(f"softmax {t}.{w} rescaled O of {self.O[t]} at block {(u, it)}")
                self.P[t][w] = (u, it)
                yield None
                self.bars["p_full", t].arrive()
            if self.nt == 1:
                # one tile per CTA: every warp (padding-only ones too) waits for the finished
                # O, writes its rows out and releases them
                yield self._wait(("o_full", t), so & 1)
                so += 1
                yield from self._read_out(t, u, nt, f"softmax {t}.{w}")
                self.bars["o_empty", t].arrive()

    def _read_out(self, t, u, n_t, who):
        if self.O[t] != (u, n_t):
            raise Race(f"{who} read O_{t} of {self.O[t]} for unit {u}")
        yield None
        if self.O[t] != (u, n_t):
            raise Race(f"O_{t} of unit {u} changed while {who} read it")
        self.o_readers += 1
        if self.o_readers == self.bars["o_empty", t].count:
            self.o_readers = 0
            self.o_read[t] = True
            self.epilogue_done.append((t, u))

    # ---------------------------------------------------------------- epilogue
    def epilogue(self):
        oe = [0] * self.nt
        for u, n in enumerate(self.units):
            for t in range(self.nt):
                if n[t] == 0:
                    continue
                yield self._wait(("o_full", t), oe[t] & 1)
                oe[t] += 1
                yield from self._read_out(t, u, n[t], "the epilogue")
                self.bars["o_empty", t].arrive()

    # ---------------------------------------------------------------- scheduler
    def run(self, rng, max_steps=400000):
        """Interleave the actors and the two async engines at random, each with a random
        speed, until everything has finished."""
        mma = [self._mma_one_tile(t) for t in range(self.nt)] if self.two_issuers else [self.mma()]
        actors = [self.producer()] + mma + ([self.epilogue()] if self.nt == 2 else []) + \
            [self.softmax(t, w) for t in range(self.nt) for w in range(WARPS)]
        na = len(actors)
        speed = [rng.uniform(0.02, 1.0) for _ in range(na + 3)]  # + tensor pipe, TMA, commits
        cond = [None] * na
        live = list(range(na))
        for _ in range(max_steps):
            runnable = [i for i in live if cond[i] is None or cond[i]()]
            if self.pipe:
                runnable.append(na)
            if self.tma:
                runnable.append(na + 1)
            ready = self.ready_commits()
            if ready:
                runnable.append(na + 2)
            if not runnable:
                if live:
                    raise Deadlock(f"{len(live)} actors blocked with nothing in flight")
                break
            i = rng.choices(runnable, weights=[speed[j] for j in runnable])[0]
            if i == na:
                self.complete_mma()
            elif i == na + 1:
                self.complete_tma(rng.randrange(len(self.tma)))
            elif i == na + 2:
                self.fire_commit(rng.choice(ready))
            else:
                try:
                    cond[i] = next(actors[i])
                except StopIteration:
                    live.remove(i)
        else:
            raise Deadlock("step limit")
        want = sorted((t, (u, it)) for u, n in enumerate(self.units)
                      for t in range(self.nt) for it in range(n[t]))
        if sorted(self.pv_done) != want:
            raise Race("not every block's P.V completed")
        if sorted(self.epilogue_done) != sorted((t, u) for u, n in enumerate(self.units)
                                                for t in range(self.nt) if n[t]):
            raise Race("not every tile's output was read out")


def random_cta(rng, separate_p=True, slots=None, drop=(), tiles=2, two_issuers=False):
    """One to five units per CTA, 0-4 key blocks per tile, random padding-only warps (warp 0
    of a tile with keys always holds a valid row)."""
    units, idle = [], []
    for _ in range(rng.randint(1, 5)):
        units.append(tuple(rng.randint(0, 4) for _ in range(tiles)))
        idle.append([set(w for w in (1, 2, 3) if rng.random() < 0.5) for _ in range(tiles)])
    return Cta(units, idle, separate_p, slots, drop, tiles, two_issuers)


def run_random(seed, **kw):
    rng = random.Random(seed)
    cta = random_cta(rng, **kw)
    cta.run(rng)
    return cta
