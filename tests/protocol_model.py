"""An executable model of the attention kernel's hand-off protocol (test helper).

The fused attention kernel coordinates its roles only through mbarriers whose
waits name a phase by its parity.  Such a wait is sound only if, when it is
made, the barrier has completed either the phase before the awaited one
(the wait blocks until the awaited phase completes) or the awaited one itself
(it passes).  If the barrier is a phase short, the parity matches the phase
before last and the wait passes early ("alias"); if it is two phases ahead,
the parity no longer matches and the wait never returns ("missed").

This model replays the roles of the kernel as written in csrc/attn_fwd.cu --
the K and V producers, the QK^T issuer, the P.V issuer and the twelve
softmax warps (three groups of four) -- as coroutines that wait, arrive and
start asynchronous operations (TMA loads, MMAs whose commits arrive when they
complete), under a random schedule with random completion delays.  Each wait
records the index of the phase it means; the scheduler flags every alias and
every missed phase, and a state where nobody can move as a deadlock.  Ring
sizes are parameters, so a test can also show that smaller rings break.
"""
from __future__ import annotations

import heapq
import random
from dataclasses import dataclass, field


class ProtocolError(AssertionError):
    pass


@dataclass
class Barrier:
    name: str
    count: int
    pending: int = 0
    completed: int = 0

    def __post_init__(self):
        self.pending = self.count

    def arrive(self):
        self.pending -= 1
        if self.pending == 0:
            self.completed += 1
            self.pending = self.count


@dataclass
class Rings:
    n_lo: int = 4          # FP4 K / e4m3 V ring slots
    n_hi: int = 1          # BF16 K / V ring slots
    s_full: int = 4        # S_FULL barriers (indexed by tile % s_full)
    p_ring: int = 8        # P_FULL barriers per softmax group
    pvc: int = 8           # P.V completion barriers
    groups: int = 3


@dataclass
class Model:
    hi: list               # BF16 flag per key tile of the query tile
    rings: Rings = field(default_factory=Rings)
    seed: int = 0
    rescale_p: float = 0.3  # chance that a softmax warp rescales O on a tile

    def __post_init__(self):
        R = self.rings
        self.rng = random.Random(self.seed)
        self.nj = len(self.hi)
        self.bars = {}
        for side in ("K", "V"):
            for kind, n in (("lo", R.n_lo), ("hi", R.n_hi)):
                for s in range(n):
                    self._bar(f"{side}{kind}_FULL{s}", 1)
                    self._bar(f"{side}{kind}_EMPTY{s}", 1)
        for s in range(R.s_full):
            self._bar(f"S_FULL{s}", 1)
        for s in range(2):
            self._bar(f"S_FREE{s}", 4)
        for g in range(R.groups):
            for u in range(R.p_ring):
                self._bar(f"P_FULL{g}_{u}", 4)
            for q in range(4):
                self._bar(f"MX{g}_{q}", 1)
        for t in range(R.pvc):
            self._bar(f"PVC{t}", 1)
        self.time = 0
        self.events = []     # (time, seq, barrier name)
        self.seq = 0
        self.async_tail = {}  # per issuing role: completion time of its last async op (in order)

    def _bar(self, name, count):
        self.bars[name] = Barrier(name, count)

    # ---------------------------------------------------------------- roles
    def _slot(self, j, side_counts):
        hi = self.hi[j]
        n = side_counts["hi" if hi else "lo"]
        slots = self.rings.n_hi if hi else self.rings.n_lo
        side_counts["hi" if hi else "lo"] += 1
        return ("hi" if hi else "lo"), n % slots, n // slots

    def producer(self, side):
        counts = {"lo": 0, "hi": 0}
        for j in range(self.nj):
            kind, slot, use = self._slot(j, counts)
            if use > 0:
                yield ("wait", f"{side}{kind}_EMPTY{slot}", use - 1)
            yield ("async", f"{side}{kind}_FULL{slot}", side)

    def qk_issuer(self):
        counts = {"lo": 0, "hi": 0}
        for j in range(self.nj):
            kind, slot, use = self._slot(j, counts)
            if j >= 2:
                yield ("wait", f"S_FREE{j & 1}", (j - 2) >> 1)
                if self.hi[j - 2]:
                    yield ("wait", f"PVC{(j - 2) % self.rings.pvc}", (j - 2) // self.rings.pvc)
            yield ("wait", f"K{kind}_FULL{slot}", use)
            yield ("async", f"K{kind}_EMPTY{slot}", "mma")
            yield ("async", f"S_FULL{j % self.rings.s_full}", "mma")

    def pv_issuer(self):
        counts = {"lo": 0, "hi": 0}
        G, P = self.rings.groups, self.rings.p_ring
        for t in range(self.nj):
            kind, slot, use = self._slot(t, counts)
            g, u = t % G, t // G
            yield ("wait", f"P_FULL{g}_{u % P}", u // P)
            yield ("wait", f"V{kind}_FULL{slot}", use)
            yield ("async", f"V{kind}_EMPTY{slot}", "mma")
            yield ("async", f"PVC{t % self.rings.pvc}", "mma")

    def softmax_warp(self, g, q):
        G, P, C = self.rings.groups, self.rings.p_ring, self.rings.pvc
        wprev = (g + G - 1) % G
        rng = random.Random(self.seed * 131 + g * 7 + q)
        for j in range(g, self.nj, G):
            yield ("wait", f"S_FULL{j % self.rings.s_full}", j // self.rings.s_full)
            yield ("arrive", f"S_FREE{j & 1}")
            if j > 0:
                yield ("wait", f"MX{wprev}_{q}", (j - 1) // G)
            if j + 1 < self.nj:
                yield ("arrive", f"MX{g}_{q}")
            if not self.hi[j] and j >= 3:
                yield ("wait", f"PVC{(j - 3) % C}", (j - 3) // C)
            if j > 0 and rng.random() < self.rescale_p:
                yield ("wait", f"PVC{(j - 1) % C}", (j - 1) // C)
            u = j // G
            yield ("arrive", f"P_FULL{g}_{u % P}")
        if self.nj > 0:   # epilogue: the last product has completed
            yield ("wait", f"PVC{(self.nj - 1) % C}", (self.nj - 1) // C)

    # ---------------------------------------------------------------- scheduler
    def run(self, max_steps=10 ** 6):
        roles = {"Kprod": self.producer("K"), "Vprod": self.producer("V"),
                 "qk": self.qk_issuer(), "pv": self.pv_issuer()}
        for g in range(self.rings.groups):
            for q in range(4):
                roles[f"sm{g}_{q}"] = self.softmax_warp(g, q)
        current = {name: next(gen, None) for name, gen in roles.items()}
        for _ in range(max_steps):
            runnable = []
            for name, act in current.items():
                if act is None:
                    continue
                if act[0] != "wait":
                    runnable.append(name)
                    continue
                b = self.bars[act[1]]
                want = act[2]
                # completed == want: blocks until the phase completes; == want + 1: passes.
                # Fewer: the parity matches an older phase (it passes now or once the
                # barrier is one phase short).  Two more: it never matches again.
                if b.completed < want:
                    raise ProtocolError(f"alias: {name} waits for phase {want} of {b.name}, "
                                        f"which has completed only {b.completed}")
                if b.completed >= want + 2:
                    raise ProtocolError(f"missed: {name} waits for phase {want} of {b.name}, "
                                        f"which has completed {b.completed}")
                if b.completed == want + 1:
                    runnable.append(name)
            if not runnable:
                if not self.events:
                    if all(a is None for a in current.values()):
                        return self.time
                    stuck = {n: a for n, a in current.items() if a is not None}
                    raise ProtocolError(f"deadlock at t={self.time}: {stuck}")
                self.time, _, bname = heapq.heappop(self.events)
                self.bars[bname].arrive()
                continue
            # either let an async operation land first, or move a random role
            if self.events and self.rng.random() < 0.3:
                self.time, _, bname = heapq.heappop(self.events)
                self.bars[bname].arrive()
                continue
            name = self.rng.choice(runnable)
            act = current[name]
            if act[0] == "arrive":
                self.bars[act[1]].arrive()
            elif act[0] == "async":
                # operations of one issuing unit complete in issue order
                unit = act[2]
                done = max(self.time, self.async_tail.get(unit, 0)) + self.rng.randint(1, 40)
                self.async_tail[unit] = done
                self.seq += 1
                heapq.heappush(self.events, (done, self.seq, act[1]))
            current[name] = next(roles[name], None)
            self.time += 1
        raise ProtocolError("step limit")
