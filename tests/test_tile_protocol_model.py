"""A model of the one-tile fine kernel's per-item synchronization, checked under random schedules (CPU).

fine_tile_kernel (block_sparse_attention_cube_b200/csrc/vsa_fine.cu) coordinates a Q/K producer (one Q
buffer, a 3-deep K ring), a V producer (a 2-deep V ring), a QK^T issuer, a PV issuer,
three softmax groups (here six half-groups: group g x query slot, each standing for the two warps of that
slot), and an epilogue warpgroup through mbarriers.  This file restates that protocol: the same barriers, the
same arrival counts (in half-group units) and the same parity waits.  An mbarrier wait by parity P succeeds
when the barrier's phase parity differs from P, so a waiter that falls a phase behind passes early.  The
tensor core completes MMAs in issue order.  Random interleavings, some with one role starved, run item
sequences of one to seven steps with random selections, and every cross-role read is checked: a row's maximum
must come from the same item, the epilogue must see the row sums of its item and an accumulator holding
exactly that item's PVs, every MMA must find its own item's Q and its own step's K or V in the buffer it
reads (copies land in any order), and nothing may deadlock.

Without the SetFree wait (a group with no step in an item can run two items ahead) or without the
once-per-item ODone barrier, the same schedules find violations; the kernel has both.  This checks the
protocol as designed, not the CUDA code; the GPU tests check the code (test_gpu_kernels.py, including
test_one_tile_kernel_with_many_items_per_cta).
"""
import random

import pytest

class Bar:
    def __init__(self, name, count):
        self.name, self.count, self.pending, self.phase = name, count, count, 0
    def arrive(self, n=1):
        self.pending -= n
        while self.pending <= 0:
            self.phase += 1
            self.pending += self.count
    def ready(self, parity):
        return (self.phase & 1) != parity

class Model:
    def __init__(self, items, seed, setfree=True, odone=True, slow=None, drop=()):
        self.rng = random.Random(seed)
        self.slow = slow
        self.drop = set(drop)          # waits left out (to show that the checks catch their absence)
        self.items = items            # list of (steps, sel) where sel[s][slot] bool
        self.setfree, self.odone = setfree, odone
        B = {}
        for b in range(3):
            B[f"SFull{b}"] = Bar(f"SFull{b}", 1)
            B[f"PFull{b}"] = Bar(f"PFull{b}", 2)      # two half-groups of the owning group
            B[f"PVDone{b}"] = Bar(f"PVDone{b}", 1)
        for ip in range(2):
            for sl in range(2):
                B[f"MReady{ip}{sl}"] = Bar(f"MReady{ip}{sl}", 1)
            B[f"Epi{ip}"] = Bar(f"Epi{ip}", 6)
            B[f"SetFree{ip}"] = Bar(f"SetFree{ip}", 1)
        B["OFree"] = Bar("OFree", 1)
        B["ODone"] = Bar("ODone", 1)
        B["QFull"], B["QEmpty"] = Bar("QFull", 1), Bar("QEmpty", 1)
        for i in range(3):
            B[f"KFull{i}"], B[f"KEmpty{i}"] = Bar(f"KFull{i}", 1), Bar(f"KEmpty{i}", 1)
        for i in range(2):
            B[f"VFull{i}"], B[f"VEmpty{i}"] = Bar(f"VFull{i}", 1), Bar(f"VEmpty{i}", 1)
        self.B = B
        self.loads = []                # copies in flight: (buffer, content, barrier), landing in any order
        self.qbuf, self.kbuf, self.vbuf = None, [None] * 3, [None] * 2
        self.fifo = []                 # tensor pipe: (kind, item, step, buf)
        self.m = {(ip, sl): None for ip in range(2) for sl in range(2)}   # value: item index
        self.l = {(ip, g, sl): None for ip in range(2) for g in range(3) for sl in range(2)}
        self.O = []                    # list of (item, step) PVs accumulated since the last release
        self.errors = []
        self.procs = {"S": self.s_issuer(), "PV": self.pv_issuer(), "EW": self.epilogue(),
                      "LQK": self.qk_producer(), "LV": self.v_producer(), "TMA": self.copies()}
        for g in range(3):
            for sl in range(2):
                self.procs[f"G{g}{sl}"] = self.half_group(g, sl)
        self.procs["T"] = self.tensor()

    # each role is a generator yielding a predicate (blocked until true) or None (a plain step)
    def wait(self, bar, parity):
        b = self.B[bar]
        return lambda: b.ready(parity)

    def qk_producer(self):
        kslot, kph = 0, 0
        for n, (steps, sel) in enumerate(self.items):
            if "QEmpty" not in self.drop:
                yield self.wait("QEmpty", (n & 1) ^ 1)
            self.loads.append(("Q", None, n, "QFull"))
            yield None
            for s in range(steps):
                yield self.wait(f"KEmpty{kslot}", kph ^ 1)
                self.loads.append(("K", kslot, (n, s), f"KFull{kslot}"))
                kslot += 1
                if kslot == 3:
                    kslot, kph = 0, kph ^ 1
                yield None

    def v_producer(self):
        vslot, vph = 0, 0
        for n, (steps, sel) in enumerate(self.items):
            for s in range(steps):
                yield self.wait(f"VEmpty{vslot}", vph ^ 1)
                self.loads.append(("V", vslot, (n, s), f"VFull{vslot}"))
                vslot += 1
                if vslot == 2:
                    vslot, vph = 0, vph ^ 1
                yield None

    def copies(self):
        while True:
            while not self.loads:
                yield lambda: bool(self.loads) or self.done_all()
                if self.done_all() and not self.loads:
                    return
            kind, slot, content, bar = self.loads.pop(self.rng.randrange(len(self.loads)))
            if kind == "Q":
                self.qbuf = content
            elif kind == "K":
                self.kbuf[slot] = content
            else:
                self.vbuf[slot] = content
            self.B[bar].arrive()
            yield None

    def s_issuer(self):
        uses = [0, 0, 0]
        kslot, kph = 0, 0
        for n, (steps, sel) in enumerate(self.items):
            yield self.wait("QFull", n & 1)
            for s in range(steps):
                b = s % 3
                if uses[b] > 0:
                    yield self.wait(f"PVDone{b}", (uses[b] - 1) & 1)
                if "KFull" not in self.drop:
                    yield self.wait(f"KFull{kslot}", kph)
                self.fifo.append(("S", n, s, (b, kslot)))
                uses[b] += 1
                kslot += 1
                if kslot == 3:
                    kslot, kph = 0, kph ^ 1
                yield None
            self.fifo.append(("QEMPTY", n, 0, None))

    def pv_issuer(self):
        waits = [0, 0, 0]
        vslot, vph = 0, 0
        for n, (steps, sel) in enumerate(self.items):
            for s in range(steps):
                b = s % 3
                if s == 0 and n > 0:
                    yield self.wait("OFree", (n - 1) & 1)
                yield self.wait(f"PFull{b}", waits[b] & 1)
                waits[b] += 1
                if "VFull" not in self.drop:
                    yield self.wait(f"VFull{vslot}", vph)
                self.fifo.append(("PV", n, s, (b, vslot)))
                vslot += 1
                if vslot == 2:
                    vslot, vph = 0, vph ^ 1
                if s == steps - 1:
                    self.fifo.append(("ODONE", n, s, b))
                yield None

    def tensor(self):
        while True:
            while not self.fifo:
                yield lambda: bool(self.fifo) or self.done_all()
                if self.done_all() and not self.fifo:
                    return
            kind, n, s, b = self.fifo.pop(0)
            if kind == "S":
                b, ks = b
                if self.qbuf != n or self.kbuf[ks] != (n, s):
                    self.errors.append(f"S({n},{s}) read Q of item {self.qbuf} and K {self.kbuf[ks]}")
                self.B[f"SFull{b}"].arrive()
                self.B[f"KEmpty{ks}"].arrive()
            elif kind == "PV":
                b, vs = b
                if self.vbuf[vs] != (n, s):
                    self.errors.append(f"PV({n},{s}) read V {self.vbuf[vs]}")
                self.O.append((n, s))
                self.B[f"PVDone{b}"].arrive()
                self.B[f"VEmpty{vs}"].arrive()
            elif kind == "QEMPTY":
                self.B["QEmpty"].arrive()
            else:
                self.B["ODone"].arrive()
            yield None

    def half_group(self, g, sl):
        n_s = 0
        for n, (steps, sel) in enumerate(self.items):
            ip, ipar = n & 1, (n >> 1) & 1
            if self.setfree and n >= 2:
                yield self.wait(f"SetFree{ip}", ((n - 2) >> 1) & 1)
            sfirst = next((s for s in range(steps) if sel[s][sl]), -1)
            have_m = False
            for s in range(steps):
                b = s % 3
                if b != g:
                    continue
                yield self.wait(f"SFull{g}", n_s & 1)
                n_s += 1
                if sel[s][sl]:
                    if s == sfirst:
                        self.m[(ip, sl)] = n
                        have_m = True
                        self.B[f"MReady{ip}{sl}"].arrive()
                        yield None
                    elif not have_m:
                        yield self.wait(f"MReady{ip}{sl}", ipar)
                        if self.m[(ip, sl)] != n:
                            self.errors.append(f"G{g}{sl} item {n} step {s} read the maximum of item {self.m[(ip, sl)]}")
                        have_m = True
                self.B[f"PFull{g}"].arrive()
                yield None
            if sfirst < 0 and g == 0:
                self.B[f"MReady{ip}{sl}"].arrive()
            self.l[(ip, g, sl)] = n
            self.B[f"Epi{ip}"].arrive()
            yield None

    def epilogue(self):
        for n, (steps, sel) in enumerate(self.items):
            ip, ipar = n & 1, (n >> 1) & 1
            if self.odone:
                yield self.wait("ODone", n & 1)
            yield self.wait(f"Epi{ip}", ipar)
            for g in range(3):
                for sl in range(2):
                    if self.l[(ip, g, sl)] != n:
                        self.errors.append(f"EW item {n} read row sums of item {self.l[(ip, g, sl)]} (group {g} slot {sl})")
            if self.setfree:
                self.B[f"SetFree{ip}"].arrive()
            yield None
            got = sorted(x for x in self.O if x[0] == n)
            if got != [(n, s) for s in range(steps)] or any(x[0] != n for x in self.O):
                self.errors.append(f"EW item {n} read O holding {self.O}")
            self.O = []
            self.B["OFree"].arrive()
            yield None

    def done_all(self):
        return all(k in ("T", "TMA") or self.finished.get(k) for k in self.procs)

    def run(self, max_steps=200000):
        self.finished = {}
        blocked_on = {}
        for _ in range(max_steps):
            runnable = []
            for k, p in self.procs.items():
                if self.finished.get(k):
                    continue
                pred = blocked_on.get(k)
                if pred is None or pred():
                    runnable.append(k)
            if not runnable:
                live = [k for k in self.procs if not self.finished.get(k)]
                if set(live) <= {"T", "TMA"}:
                    return
                self.errors.append("deadlock: " + ", ".join(live))
                return
            if self.slow in runnable and len(runnable) > 1 and self.rng.random() < 0.97:
                runnable = [x for x in runnable if x != self.slow]
            k = self.rng.choice(runnable)
            try:
                nxt = next(self.procs[k])
                blocked_on[k] = nxt
            except StopIteration:
                self.finished[k] = True
                blocked_on.pop(k, None)
            if all(self.finished.get(x) for x in self.procs if x not in ("T", "TMA")) and not self.fifo \
                    and not self.loads:
                return
        self.errors.append("step limit")

def random_items(rng, n_items):
    items = []
    for _ in range(n_items):
        steps = rng.choice([1, 1, 2, 2, 3, 4, 5, 7])
        sel = [[rng.random() < 0.8, rng.random() < 0.8] for _ in range(steps)]
        items.append((steps, sel))
    return items



def random_items(rng, n_items):
    items = []
    for _ in range(n_items):
        steps = rng.choice([1, 1, 2, 2, 3, 4, 5, 7])
        sel = [[rng.random() < 0.8, rng.random() < 0.8] for _ in range(steps)]
        items.append((steps, sel))
    return items


ROLES = ["S", "PV", "EW", "T", "LQK", "LV", "TMA"] + [f"G{g}{sl}" for g in range(3) for sl in range(2)] + [None]


def _violations(trials, setfree=True, odone=True, drop=()):
    bad = []
    for t in range(trials):
        rng = random.Random(t)
        m = Model(random_items(rng, rng.randint(1, 12)), seed=t, setfree=setfree, odone=odone,
                  slow=rng.choice(ROLES), drop=drop)
        m.run()
        if m.errors:
            bad.append((t, m.errors[:2]))
    return bad


def test_protocol_holds_under_random_schedules():
    bad = _violations(400)
    assert not bad, bad[:3]


def test_the_model_finds_the_run_ahead_race_without_setfree():
    assert _violations(200, setfree=False)


def test_the_model_finds_an_early_output_read_without_the_once_per_item_barrier():
    assert _violations(200, odone=False)


@pytest.mark.parametrize("wait", ["QEmpty", "KFull", "VFull"])
def test_the_model_finds_stale_operands_without_each_load_wait(wait):
    assert _violations(200, drop=(wait,))
