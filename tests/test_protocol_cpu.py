"""Discrete-event check of the convolution kernel's mbarrier protocol (CPU only).

The tensor-core kernel (smc_conv_tc.cu) hands A units, W slices, gather
indices and accumulators between its warp roles through mbarriers that are
waited on by phase parity.  A parity wait cannot tell phase k from phase k + 2,
so the protocol is only correct if no wait can ever be two phases ahead of its
barrier, no ring slot is overwritten while it is read, and every role
terminates.  This test runs one CTA's roles as coroutines over a random item
list with random latencies and checks exactly that:

* barriers follow the hardware rule: try_wait.parity(P) passes iff the current
  phase's parity differs from P; each passing wait is also checked against the
  phase it logically waits for (the completed phase count must be exactly that
  phase + 1);
* slot contents: a consumer finds the unit / stage it expects in the slot, and
  a producer never refills a slot a consumer is still reading;
* the run ends (no deadlock), every unit is multiplied once, every item's
  output is stored once, the last item's columns split between the epilogue
  warps and the helper warps.

The roles mirror the kernel: W loader (one lane), index prefetcher (one lane,
sparse mode), NQ gather groups of WPS warps (one arrival per lane), two MMA
warps sharing one in-order tensor pipe (commits arrive when the warp's earlier
MMAs complete), the epilogue warps, and the four helper warps that store half
of the last item after a one-phase barrier.  The kernel's compile-time rule
NW * G <= NA is what keeps the MMA warps' A-slot waits unambiguous; a
configuration that breaks it must be caught here.
"""
import heapq
import random

import pytest

TAPS = 27


class Bar:
    def __init__(self, name, count):
        self.name, self.count = name, count
        self.pending, self.tx, self.phase = count, 0, 0

    def arrive(self, n=1):
        self.pending -= n
        assert self.pending >= 0, (self.name, "too many arrivals")
        self._check()

    def expect_tx(self, b):
        self.tx += b

    def complete_tx(self, b):
        self.tx -= b
        assert self.tx >= 0, (self.name, "tx underflow")
        self._check()

    def _check(self):
        if self.pending == 0 and self.tx == 0:
            self.phase += 1
            self.pending = self.count

    def passes(self, parity):
        return (self.phase & 1) != parity


class Cta:
    """One CTA of the persistent kernel over a static list of work items."""

    def __init__(self, rng, items, G, NA, NW, NQ, WPS, NBUF, kbt, dense):
        self.rng, self.items = rng, items
        self.G, self.NA, self.NW, self.NQ, self.WPS, self.NBUF = G, NA, NW, NQ, WPS, NBUF
        self.kbt, self.dense = kbt, dense
        self.t = 0
        self.seq = 0
        self.events = []
        self.afull = [Bar(f"afull{i}", 1 if dense else WPS * 32) for i in range(NA)]
        self.aempty = [Bar(f"aempty{i}", 1) for i in range(NA)]
        self.ifull = [Bar(f"ifull{i}", 1) for i in range(NA)]
        self.iempty = [Bar(f"iempty{i}", WPS) for i in range(NA)]
        self.wfull = [Bar(f"wfull{i}", 1) for i in range(NW)]
        self.wempty = [Bar(f"wempty{i}", 2) for i in range(NW)]
        self.tfull = [Bar(f"tfull{i}", 2) for i in range(2)]
        self.tempty = [Bar(f"tempty{i}", 128) for i in range(2)]
        self.info = [Bar(f"info{i}", 1) for i in range(2)]
        self.lastdone = Bar("lastdone", 2)
        self.acc_info = [None, None]
        self.a_content = [None] * NA
        self.a_reading = [0] * NA
        self.i_content = [None] * NA
        self.w_content = [None] * NW
        self.w_reading = [0] * NW
        self.tensor_tail = 0          # the tensor pipe runs MMAs in issue order
        self.warp_done = [0, 0]       # completion time of each MMA warp's last MMA
        self.consumed = 0
        self.stored = []              # (item, half) pairs written

    # ---- event machinery ----
    def delay(self, lo, hi):
        return self.rng.randint(lo, hi)

    def at(self, when, fn):
        self.seq += 1
        heapq.heappush(self.events, (when, self.seq, fn))

    def run(self, procs, limit=2_000_000):
        state = [[p, None] for p in procs]
        steps = 0
        while True:
            progressed = False
            for st in state:
                gen, cond = st
                if gen is None:
                    continue
                while True:
                    if cond is not None:
                        if cond[0] == "wait":
                            _, bar, parity, logical = cond
                            if not bar.passes(parity):
                                break
                            assert bar.phase == logical + 1, (bar.name, "phase", bar.phase,
                                                              "waited for", logical)
                        elif self.t < cond[1]:
                            break
                    try:
                        cond = next(gen)
                    except StopIteration:
                        st[0] = None
                        progressed = True
                        break
                    if cond[0] == "sleep":
                        cond = ("sleep", self.t + cond[1])
                    st[1] = cond
                    progressed = True
            if all(st[0] is None for st in state):
                return
            if not progressed:
                times = [e[0] for e in self.events[:1]]
                times += [st[1][1] for st in state if st[0] is not None and st[1][0] == "sleep"]
                if not times:
                    stuck = [st[1][1].name for st in state if st[0] is not None and st[1][0] == "wait"]
                    raise RuntimeError(f"deadlock: {stuck}")
                self.t = max(self.t, min(times))
                while self.events and self.events[0][0] <= self.t:
                    heapq.heappop(self.events)[2]()
            steps += 1
            assert steps < limit, "step limit"

    # ---- the walk every role makes ----
    def item(self, j):
        if j >= len(self.items):
            return None
        masks = self.items[j]
        allm = 0
        for m in masks:
            allm |= m
        rot = 0 if self.dense else (j * 7) % TAPS
        taps = [t for t in ((rot + i) % TAPS for i in range(TAPS)) if (allm >> t) & 1]
        return {"j": j, "masks": masks, "taps": taps}

    def units(self, it):
        """(stage, tile) of every unit of the item, in the kernel's numbering order."""
        out = []
        for tap in it["taps"]:
            for kb in range(self.kbt):
                out.append([k for k in range(self.G) if (it["masks"][k] >> tap) & 1])
        return out

    # ---- roles ----
    def w_loader(self):
        s, j = 0, 0
        while (it := self.item(j)) is not None:
            j += 1
            for _ in self.units(it):
                ws = s % self.NW
                yield ("wait", self.wempty[ws], ((s // self.NW) & 1) ^ 1, s // self.NW - 1)
                assert self.w_reading[ws] == 0, ("W slot refilled while read", ws)
                self.w_content[ws] = ("landing", s)
                b = self.wfull[ws]
                b.expect_tx(1)
                b.arrive()

                def land(b=b, ws=ws, s=s):
                    self.w_content[ws] = ("ready", s)
                    b.complete_tx(1)
                self.at(self.t + self.delay(50, 1200), land)
                s += 1
                yield ("sleep", self.delay(1, 5))

    def idx_prefetcher(self):
        u, j = 0, 0
        while (it := self.item(j)) is not None:
            j += 1
            if self.dense:
                continue
            for tiles in self.units(it):
                for _ in tiles:
                    slot = u % self.NA
                    yield ("wait", self.iempty[slot], ((u // self.NA) & 1) ^ 1, u // self.NA - 1)
                    b = self.ifull[slot]
                    b.expect_tx(1)
                    b.arrive()

                    def land(b=b, slot=slot, u=u):
                        self.i_content[slot] = u
                        b.complete_tx(1)
                    self.at(self.t + self.delay(50, 1500), land)
                    u += 1
                    yield ("sleep", self.delay(1, 5))

    def gather_warp(self, grp, wq, helper):
        u, j, last, n = 0, 0, None, 0
        while (it := self.item(j)) is not None:
            j += 1
            last, n = it, n + 1
            for tiles in self.units(it):
                mine = [(u + i, k) for i, k in enumerate(tiles) if (u + i) % self.NQ == grp]
                u += len(tiles)
                assert len(mine) <= 1, "two units of one stage in one gather group"
                for my, _k in mine:
                    slot, ph = my % self.NA, (my // self.NA) & 1
                    if self.dense:
                        if wq == 0:
                            yield ("wait", self.aempty[slot], ph ^ 1, my // self.NA - 1)
                            assert self.a_reading[slot] == 0, ("A slot refilled while read", slot)
                            self.a_content[slot] = ("landing", my)
                            b = self.afull[slot]
                            b.expect_tx(1)
                            b.arrive()

                            def land(b=b, slot=slot, my=my):
                                self.a_content[slot] = ("ready", my)
                                b.complete_tx(1)
                            self.at(self.t + self.delay(100, 2000), land)
                        continue
                    yield ("wait", self.ifull[slot], ph, my // self.NA)
                    assert self.i_content[slot] == my, ("index block", self.i_content[slot], my)
                    yield ("sleep", self.delay(1, 20))
                    self.iempty[slot].arrive()
                    yield ("wait", self.aempty[slot], ph ^ 1, my // self.NA - 1)
                    assert self.a_reading[slot] == 0, ("A slot refilled while read", slot)
                    self.a_content[slot] = ("landing", my)

                    # one arrival per lane, made when that lane's copies land
                    def land(slot=slot, my=my):
                        b = self.afull[slot]
                        b.arrive(32)
                        if b.phase == my // self.NA + 1:
                            self.a_content[slot] = ("ready", my)
                    self.at(self.t + self.delay(100, 2500), land)
                    yield ("sleep", self.delay(10, 60))
        if helper and n:
            # store the second half of the last item once its MMAs are done
            yield ("wait", self.lastdone, 0, 0)
            a = (n - 1) % self.NBUF
            assert self.acc_info[a] is not None and self.acc_info[a]["j"] == last["j"], "helper item"
            yield ("sleep", self.delay(50, 800))
            if wq == 0 and grp == 0:
                self.stored.append((last["j"], 1))

    def mma_warp(self, mine):
        u, s, j, acc_iter = 0, 0, 0, 0
        while True:
            it = self.item(j)
            j += 1
            a, use = acc_iter % self.NBUF, acc_iter // self.NBUF
            yield ("wait", self.tempty[a], (use & 1) ^ 1, use - 1)
            if mine == 0:
                self.acc_info[a] = it
                self.info[a].arrive()
            if it is None:
                return
            for tiles in self.units(it):
                ws = s % self.NW
                yield ("wait", self.wfull[ws], (s // self.NW) & 1, s // self.NW)
                assert self.w_content[ws] == ("ready", s), ("W slot", self.w_content[ws], s)
                own = [(u + i, k) for i, k in enumerate(tiles) if (k & 1) == mine]
                u += len(tiles)
                assert len(own) <= 1
                self.w_reading[ws] += 1
                for my, _k in own:
                    slot = my % self.NA
                    yield ("wait", self.afull[slot], (my // self.NA) & 1, my // self.NA)
                    assert self.a_content[slot] == ("ready", my), ("A slot", self.a_content[slot], my)
                    self.a_reading[slot] += 1
                    # the MMAs queue on the shared tensor pipe; the issuing
                    # thread is held until they are accepted
                    done = max(self.tensor_tail, self.t) + self.delay(64, 520)
                    self.tensor_tail = done
                    self.warp_done[mine] = done
                    yield ("sleep", max(0, done - 500 - self.t) + self.delay(1, 30))

                    def release(slot=slot):
                        self.a_reading[slot] -= 1
                        self.consumed += 1
                        self.aempty[slot].arrive()
                    self.at(max(self.t, self.warp_done[mine]) + self.delay(20, 150), release)

                def w_release(ws=ws):
                    self.w_reading[ws] -= 1
                    self.wempty[ws].arrive()
                self.at(max(self.t, self.warp_done[mine]) + self.delay(20, 150), w_release)
                s += 1
            when = max(self.t, self.warp_done[mine]) + self.delay(20, 150)
            self.at(when, lambda a=a: self.tfull[a].arrive())
            if self.item(j) is None:
                self.at(when + 1, self.lastdone.arrive)
            acc_iter += 1

    def epilogue(self):
        acc_iter = 0
        while True:
            a, use = acc_iter % self.NBUF, acc_iter // self.NBUF
            yield ("wait", self.info[a], use & 1, use)
            it = self.acc_info[a]
            if it is None:
                return
            yield ("wait", self.tfull[a], use & 1, use)
            yield ("sleep", self.delay(100, 1500))
            last = it["j"] == len(self.items) - 1
            self.stored.append((it["j"], 0))
            if not last:
                self.stored.append((it["j"], 1))
            self.tempty[a].arrive(128)
            acc_iter += 1


def random_items(rng, n, G, dense, ptap):
    items = []
    for _ in range(n):
        masks = []
        for k in range(G):
            if dense:
                masks.append(1 << 13)
                continue
            r = rng.random()
            if r < 0.1:
                m = 1 << 13
            elif r < 0.15 and k > 0:
                m = 0  # past the last tile
            else:
                m = (1 << 13) | sum(1 << t for t in range(TAPS) if rng.random() < ptap)
            masks.append(m)
        items.append(tuple(masks))
    return items


def run(seed, G, NA, NW, NQ, WPS, NBUF, kbt, dense, n_items, ptap):
    rng = random.Random(seed)
    items = random_items(rng, n_items, G, dense, ptap)
    cta = Cta(rng, items, G, NA, NW, NQ, WPS, NBUF, kbt, dense)
    procs = [cta.w_loader(), cta.idx_prefetcher(), cta.mma_warp(0), cta.mma_warp(1), cta.epilogue()]
    for g in range(NQ):
        for w in range(WPS):
            procs.append(cta.gather_warp(g, w, helper=(g * WPS + w) < 4))
    cta.run(procs)
    units = sum(len(tiles) for it in (cta.item(j) for j in range(len(items))) for tiles in cta.units(it))
    assert cta.consumed == units, (cta.consumed, units)
    assert sorted(cta.stored) == sorted((j, h) for j in range(len(items)) for h in (0, 1)), "stores"


# The kernel's launch configurations: G, NA, NW, NQ, WPS, NBUF, 64-channel stages per tap, K = 1.
CONFIGS = [
    (2, 4, 2, 2, 4, 2, 1, False),    # 128-column, two tiles, 128-channel units (uniform128)
    (1, 4, 2, 2, 4, 2, 1, False),    # same, one tile per item
    (2, 10, 3, 5, 2, 2, 2, False),   # 128-column, 64-channel units
    (2, 12, 2, 6, 2, 2, 1, False),   # 64-column (shells512)
    (1, 5, 2, 5, 2, 2, 1, False),    # 64-column tap pairs (uniform64)
    (2, 9, 2, 3, 4, 1, 8, False),    # 256-column, one accumulator set (resblock64 3x3x3)
    (1, 2, 2, 2, 4, 2, 4, True),     # 256-column K = 1 (resblock64 1x1x1)
]


@pytest.mark.parametrize("cfg", CONFIGS)
def test_protocol_configurations(cfg):
    G, NA, NW, NQ, WPS, NBUF, kbt, dense = cfg
    assert NA % NQ == 0 and NQ >= G and NW * G <= NA  # the kernel's compile-time rules
    for seed in range(6):
        for ptap in (0.03, 0.3, 0.9):
            run(seed, G, NA, NW, NQ, WPS, NBUF, kbt, dense, 1 + (seed * 5) % 9, ptap)


def test_protocol_check_catches_drift_aliasing():
    # NW * G > NA lets one MMA warp wait on an A slot two phases ahead; the
    # parity wait then passes on a stale phase, which the check must report
    caught = False
    for seed in range(30):
        try:
            run(seed, 2, 4, 3, 2, 4, 2, 1, False, 6, 0.9)
        except AssertionError as e:
            caught = caught or ("afull" in str(e) and "phase" in str(e))
    assert caught


@pytest.mark.parametrize("planted", ["helper skips lastdone", "W wait only for own units",
                                     "epilogue skips tfull"])
def test_protocol_check_catches_planted_mistakes(planted):
    # the simulation itself must fail when a wait the kernel relies on is removed
    import inspect
    import sys
    src = inspect.getsource(sys.modules[__name__])
    edits = {
        "helper skips lastdone": ('            yield ("wait", self.lastdone, 0, 0)\n', ""),
        "W wait only for own units": (
            '                yield ("wait", self.wfull[ws], (s // self.NW) & 1, s // self.NW)\n'
            '                assert self.w_content[ws] == ("ready", s), ("W slot", self.w_content[ws], s)\n'
            '                own = [(u + i, k) for i, k in enumerate(tiles) if (k & 1) == mine]',
            '                own = [(u + i, k) for i, k in enumerate(tiles) if (k & 1) == mine]\n'
            '                if own:\n'
            '                    yield ("wait", self.wfull[ws], (s // self.NW) & 1, s // self.NW)\n'
            '                    assert self.w_content[ws] == ("ready", s), ("W slot", self.w_content[ws], s)'),
        "epilogue skips tfull": ('            yield ("wait", self.tfull[a], use & 1, use)\n', ""),
    }
    a, b = edits[planted]
    assert a in src
    ns = {}
    exec(compile(src.replace(a, b, 1), "planted", "exec"), ns)
    failures = 0
    for cfg in CONFIGS[:4]:
        G, NA, NW, NQ, WPS, NBUF, kbt, dense = cfg
        for seed in range(4):
            try:
                ns["run"](seed, G, NA, NW, NQ, WPS, NBUF, kbt, dense, 1 + (seed * 5) % 9, 0.3)
            except (AssertionError, RuntimeError):
                failures += 1
    assert failures > 0, planted
