"""Discrete-event model of the mbarrier protocol of the block-sparse attention
kernel (sparse_attn_kernel in csrc/k_attn.cu), for checking it on the CPU.

Roles, as in the kernel: the producer (warp 0: per item a Q load, then one step
record per step and the K loads of that step), the S-MMA issuer (warp 1), the
PV-MMA issuer (warp 10), the V producer (warp 11) and two softmax groups taking
alternate steps.  Barriers carry the kernel's arrival counts (per-warp counts
folded into one arrival per group), TMA transaction bytes, and phases; a
parity wait succeeds exactly when the mbarrier's current phase has the other
parity, as the hardware's does.  TMA loads and MMAs complete after random
delays and the roles advance in random order, so each run is one interleaving.

Checks: every role finishes (no deadlock); every parity wait succeeds on
exactly the phase it names (neither early nor lapped); no K/V stage, step
record slot or TMEM S buffer is reused before its previous user is done; every
MMA finds its operands loaded.  With `check_epilogue` the epilogue's wait on
the O-complete barriers (one per item parity) is the kernel's parity wait and
is checked like the others; without it, it is modelled as a wait for its own
item's phase, so the rest of the protocol is checked on its own.  A variant
with a single O-complete barrier (`single_o_full`) reproduces the ordering gap
that the per-parity pair closes."""
import random

RING, META = 3, 8


class Barrier:
    def __init__(self, name, count):
        self.name, self.count = name, count
        self.phase = 0            # completed phases
        self.arrived = 0
        self.tx = 0

    def _complete(self):
        if self.arrived == self.count and self.tx == 0:
            self.phase += 1
            self.arrived = 0

    def arrive(self):
        self.arrived += 1
        assert self.arrived <= self.count, f"over-arrival on {self.name}"
        self._complete()

    def arrive_expect_tx(self, nbytes):
        self.tx += nbytes
        self.arrive()

    def complete_tx(self, nbytes):
        self.tx -= nbytes
        assert self.tx >= 0, f"negative transaction count on {self.name}"
        self._complete()

    def parity_done(self, parity):
        return (self.phase & 1) != parity


class Model:
    def __init__(self, items, rng, check_epilogue, single_o_full=False):
        self.items, self.rng, self.check_epilogue = items, rng, check_epilogue
        self.single_o_full = single_o_full
        self.t = 0
        self.events = []
        mk = Barrier
        self.k_full = [mk(f"k_full{i}", 1) for i in range(RING)]
        self.v_full = [mk(f"v_full{i}", 1) for i in range(RING)]
        self.s_full = [mk(f"s_full{i}", 1) for i in range(RING)]
        self.pv_buf = [mk(f"pv_buf{i}", 1) for i in range(RING)]
        self.meta_full = [mk(f"meta_full{i}", 1) for i in range(META)]
        self.meta_empty = [mk(f"meta_empty{i}", 1) for i in range(META)]  # 4 warps of a group
        self.q_full, self.q_empty = mk("q_full", 1), mk("q_empty", 1)
        self.p_full = [mk(f"p_full{i}", 1) for i in range(4)]
        self.o_full = [mk(f"o_full{i}", 1) for i in range(1 if single_o_full else 2)]
        self.o_empty = mk("o_empty", 1)
        self.m_full = [mk(f"m_full{i}", 1) for i in range(2)]
        self.l_full = [mk(f"l_full{i}", 1) for i in range(2)]
        self.meta = [None] * META
        self.done = set()          # ("K"|"V"|"S"|"PV", step)
        self.readers = {}          # step -> roles that copied its record

    def later(self, fn, lo=1, hi=40):
        self.events.append((self.t + self.rng.randint(lo, hi), fn))

    def wait(self, bar, parity, phase, exact=True):
        while not bar.parity_done(parity):
            yield
        if exact:
            assert bar.phase == phase + 1, (
                f"{bar.name}: wait for phase {phase} succeeded at phase {bar.phase}")

    def read(self, n, who):
        r = self.meta[n % META]
        assert r is not None and r["n"] == n, f"{who} read a stale record for step {n}"
        self.readers.setdefault(n, set()).add(who)
        return r

    def o_slot(self, seq):
        """The O-complete barrier of item `seq`."""
        return 0 if self.single_o_full else seq & 1

    # ------------------------------------------------------------------ roles
    def producer(self):
        m = 0

        def emit(rec):
            nonlocal m
            sm, s3 = m % META, m % RING
            yield from self.wait(self.meta_empty[sm], ((m // META) & 1) ^ 1, m // META - 1)
            if m >= RING:
                yield from self.wait(self.s_full[s3], ((m - RING) // RING) & 1, (m - RING) // RING)
                assert ("S", m - RING) in self.done, "K stage reused before its S MMA finished"
            if m >= META:
                assert {"G", "S", "PV", "V"} <= self.readers.get(m - META, set()), \
                    f"record slot of step {m - META} rewritten before every reader copied it"
            self.meta[sm] = dict(rec, n=m)
            self.meta_full[sm].arrive()
            nb = max(rec["nb"], 0)
            kf = self.k_full[s3]
            kf.arrive_expect_tx(nb)
            step = m
            if nb:
                self.later(lambda: (kf.complete_tx(nb), self.done.add(("K", step))))
            else:
                self.done.add(("K", step))
            m += 1

        for seq, steps in enumerate(self.items):
            if seq > 0:
                yield from self.wait(self.q_empty, (seq - 1) & 1, seq - 1)
            self.q_full.arrive_expect_tx(2)
            self.later(lambda: self.q_full.complete_tx(2))
            for j, nb in enumerate(steps):
                yield from emit({"nb": nb, "first": j == 0, "last": j == len(steps) - 1,
                                 "seq": seq})
        end = {"nb": -1, "first": False, "last": False, "seq": 0}
        yield from emit(end)        # one end record per softmax group
        yield from emit(end)

    def s_issuer(self):
        n = 0
        while True:
            b = n % RING
            yield from self.wait(self.k_full[b], (n // RING) & 1, n // RING)
            r = self.read(n, "S")
            if r["nb"] < 0:
                return
            if n >= RING:
                yield from self.wait(self.pv_buf[b], ((n - RING) // RING) & 1, (n - RING) // RING)
                assert ("PV", n - RING) in self.done, "S buffer reused before its PV finished"
            if r["first"]:
                yield from self.wait(self.q_full, r["seq"] & 1, r["seq"])
            assert r["nb"] == 0 or ("K", n) in self.done, "S MMA before its K landed"

            def finish(b=b, n=n, last=r["last"]):
                self.done.add(("S", n))
                self.s_full[b].arrive()
                if last:
                    self.q_empty.arrive()
            self.later(finish, 5, 60)
            n += 1

    def pv_issuer(self):
        n = 0
        while True:
            b = n % RING
            yield from self.wait(self.meta_full[n % META], (n // META) & 1, n // META)
            r = self.read(n, "PV")
            if r["nb"] < 0:
                return
            yield from self.wait(self.p_full[n & 3], (n >> 2) & 1, n >> 2)
            if r["first"] and r["seq"] > 0:
                yield from self.wait(self.o_empty, (r["seq"] - 1) & 1, r["seq"] - 1)
            yield from self.wait(self.v_full[b], (n // RING) & 1, n // RING)
            assert r["nb"] == 0 or ("V", n) in self.done, "PV MMA before its V landed"

            def finish(b=b, n=n, last=r["last"], seq=r["seq"]):
                # the kernel commits O complete before the step's pv_buf, and
                # commits arrive in issue order
                self.done.add(("PV", n))
                if last:
                    self.o_full[self.o_slot(seq)].arrive()
                self.pv_buf[b].arrive()
            self.later(finish, 5, 60)
            n += 1

    def v_producer(self):
        n = 0
        while True:
            b = n % RING
            yield from self.wait(self.meta_full[n % META], (n // META) & 1, n // META)
            r = self.read(n, "V")
            if r["nb"] < 0:
                return
            if n >= RING:
                yield from self.wait(self.pv_buf[b], ((n - RING) // RING) & 1, (n - RING) // RING)
                assert ("PV", n - RING) in self.done, "V stage reused before its PV finished"
            nb = max(r["nb"], 0)
            vf = self.v_full[b]
            vf.arrive_expect_tx(nb)
            step = n
            if nb:
                self.later(lambda vf=vf, nb=nb, step=step: (vf.complete_tx(nb),
                                                            self.done.add(("V", step))))
            else:
                self.done.add(("V", step))
            n += 1

    def softmax_group(self, g):
        n = g
        while True:
            sm = n % META
            yield from self.wait(self.meta_full[sm], (n // META) & 1, n // META)
            r = self.read(n, "G")
            self.meta_empty[sm].arrive()
            if r["nb"] < 0:
                return
            yield from self.wait(self.s_full[n % RING], (n // RING) & 1, n // RING)
            if n > 0:
                yield from self.wait(self.m_full[(n - 1) & 1], ((n - 1) >> 1) & 1, (n - 1) >> 1)
            if r["last"] and not r["first"]:
                yield from self.wait(self.l_full[(n - 1) & 1], ((n - 1) >> 1) & 1, (n - 1) >> 1)
            self.m_full[n & 1].arrive()
            for _ in range(self.rng.randint(0, 3)):     # the exponentials
                yield
            self.l_full[n & 1].arrive()
            if n > 0 and not r["first"] and self.rng.random() < 0.3:   # lazy O rescale
                p = n - 1
                yield from self.wait(self.pv_buf[p % RING], (p // RING) & 1, p // RING)
                assert ("PV", p) in self.done
            self.p_full[n & 3].arrive()
            if r["last"]:
                ob = self.o_full[self.o_slot(r["seq"])]
                ph = r["seq"] if self.single_o_full else r["seq"] >> 1
                if self.check_epilogue:      # the kernel's parity wait, checked
                    yield from self.wait(ob, ph & 1, ph)
                else:                        # an ordered wait for this item's phase
                    while ob.phase < ph + 1:
                        yield
                assert ("PV", n) in self.done, "epilogue read O before its last PV finished"
                self.o_empty.arrive()
            n += 2

    # ------------------------------------------------------------------ driver
    def state(self, live):
        bars = (self.k_full + self.v_full + self.s_full + self.pv_buf + self.meta_full +
                self.meta_empty + self.p_full + self.m_full + self.l_full +
                self.o_full + [self.q_full, self.q_empty, self.o_empty])
        return (len(live),) + tuple((b.phase, b.arrived, b.tx) for b in bars)

    def run(self):
        live = {"producer": self.producer(), "S": self.s_issuer(), "PV": self.pv_issuer(),
                "V": self.v_producer(), "G0": self.softmax_group(0),
                "G1": self.softmax_group(1)}
        still, last = 0, None
        while live:
            self.t += 1
            due = [e for e in self.events if e[0] <= self.t]
            self.events = [e for e in self.events if e[0] > self.t]
            for _, fn in due:
                fn()
            names = list(live)
            self.rng.shuffle(names)
            for name in names:
                try:
                    next(live[name])
                except StopIteration:
                    del live[name]
            now = self.state(live)
            still = still + 1 if (not self.events and now == last) else 0
            last = now
            assert still < 50, f"deadlock: {sorted(live)} blocked at t={self.t}"


def random_items(rng):
    """Items (query-tile pairs) as lists of per-step key-block counts: empty
    items (one step, no blocks), single-step items and longer ones whose last
    step may hold one block."""
    items = []
    for _ in range(rng.choice([1, 1, 2, 3, 5, 8, 13])):
        if rng.random() < 0.1:
            items.append([0])
            continue
        k = rng.choice([1, 1, 2, 3, 4, 7, 12, 20])
        items.append([2] * (k - 1) + [rng.choice([1, 2])])
    return items


def run_schedules(count, seed, check_epilogue, single_o_full=False):
    rng = random.Random(seed)
    for _ in range(count):
        Model(random_items(rng), random.Random(rng.random()), check_epilogue,
              single_o_full).run()
