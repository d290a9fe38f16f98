"""Discrete-event model of a warp-specialised kernel's synchronisation: mbarriers, TMA copies, the tensor pipe and the
roles' own accesses to shared memory and TMEM. It checks a kernel's protocol on the CPU, not its arithmetic.

A role is a generator of actions, written to follow the role's loop in the kernel:
  ("wait", bar, k)         block until the barrier's parity test for phase k passes (hardware rule: it passes while
                           completed % 2 != k % 2); passing with any count other than k + 1 completed phases is an error
                           (a stale or skipped phase), and so is waiting forever (a deadlock)
  ("arrive", bar[, n])     n arrivals; a warpgroup that arrives with all its threads is modelled as one arrival
  ("expect", bar, units)   arrive with an expected transaction count
  ("tma", bar, units, r)   asynchronous copy into region r that completes the transactions after a random delay
  ("store", bar, r)        asynchronous copy out of region r that arrives on bar once it has read r
  ("mma", reads, writes)   asynchronous tensor-pipe operation, in issue order
  ("commit", bar)          arrive on bar once every tensor operation issued so far has completed
  ("read", r) / ("write", r)     a role's own access
  ("put", r, v) / ("get", r, v)  a role's own write of a tagged value, and a read that expects that value
A role's access to a region that an asynchronous copy or tensor operation may still write (or, for a write, still
read) is an error. With pipe_overlap, consecutive tensor operations may run concurrently, and a write to a region
that an earlier operation may still read is an error too. Roles are scheduled at random, with random stalls, so
that many interleavings are tried.
"""
import random


class Barrier:
    def __init__(self, name, count):
        self.name, self.count = name, count
        self.pending, self.tx, self.completed = count, 0, 0

    def settle(self):
        if self.pending == 0 and self.tx == 0:
            self.completed += 1
            self.pending = self.count


class Model:
    def __init__(self, seed, max_delay=5, pipe_overlap=False, stall_p=0.05, stall_max=200):
        self.rng = random.Random(seed)
        self.max_delay = max_delay
        self.pipe_overlap = pipe_overlap
        self.stall_p, self.stall_max = stall_p, stall_max
        self.bars, self.roles, self.values = {}, {}, {}
        self.events = []  # (time, sequence, callback)
        self.t = self.seq = 0
        self.errors = []
        self.pipe_last_start, self.pipe_last_done = -1, 0
        self.pipe_reads, self.pipe_writes = {}, {}  # region -> completion times of tensor operations
        self.copy_reads, self.copy_writes = {}, {}  # region -> completion times of TMA copies
        self.op_done = []

    # ------------------------------------------------------------------------------------------------ set-up
    def bar(self, name, count=1):
        self.bars[name] = Barrier(name, count)

    def err(self, msg):
        if len(self.errors) < 20:
            self.errors.append(f"t={self.t}: {msg}")

    # ------------------------------------------------------------------------------------------------ helpers
    def _later(self, dt, fn):
        self.seq += 1
        self.events.append((self.t + dt, self.seq, fn))

    def _live(self, table, reg, after=None):
        t = self.t if after is None else after
        return [d for d in table.get(reg, []) if d > t]

    def _access(self, role, kind, reg):
        if self._live(self.copy_writes, reg) or self._live(self.pipe_writes, reg):
            self.err(f"{role}: {kind} of {reg} while an asynchronous write to it may be in flight")
        if kind == "write" and (self._live(self.copy_reads, reg) or self._live(self.pipe_reads, reg)):
            self.err(f"{role}: write of {reg} while an asynchronous read of it may be in flight")

    def _arrive(self, bar, n=1):
        B = self.bars[bar]
        B.pending -= n
        if B.pending < 0:
            self.err(f"{bar}: more arrivals than its count")
        B.settle()

    def _advance(self, force=False):
        if not self.events:
            self.t += 1
            return
        self.events.sort()
        if not force and self.events[0][0] > self.t + 1:
            self.t += 1
            return
        self.t = max(self.t, self.events[0][0])
        due = [e for e in self.events if e[0] <= self.t]
        self.events = [e for e in self.events if e[0] > self.t]
        for _, _, fn in due:
            fn()

    # ------------------------------------------------------------------------------------------------ actions
    def _do(self, role, act):
        kind = act[0]
        if kind == "arrive":
            self._arrive(act[1], act[2] if len(act) > 2 else 1)
        elif kind == "expect":
            self.bars[act[1]].tx += act[2]
            self._arrive(act[1])
        elif kind == "tma":
            _, bar, units, reg = act
            self._access(role, "write", reg)
            d = self.rng.randint(1, 3 * self.max_delay)
            self.copy_writes.setdefault(reg, []).append(self.t + d)

            def land(bar=bar, units=units):
                self.bars[bar].tx -= units
                self.bars[bar].settle()
            self._later(d, land)
        elif kind == "store":
            _, bar, reg = act
            self._access(role, "read", reg)
            d = self.rng.randint(1, 2 * self.max_delay)
            self.copy_reads.setdefault(reg, []).append(self.t + d)
            self._later(d, lambda bar=bar: self._arrive(bar))
        elif kind == "mma":
            _, reads, writes = act
            for r in reads:
                if self._live(self.copy_writes, r):
                    self.err(f"{role}: tensor operation reads {r} while a copy into it may be in flight")
            start = max(self.t, self.pipe_last_start + 1) if self.pipe_overlap else max(self.t, self.pipe_last_done)
            done = max(start + self.rng.randint(1, self.max_delay), self.pipe_last_done + 1)
            for w in writes:
                if self._live(self.pipe_reads, w, after=start):
                    self.err(f"{role}: tensor operation writes {w} while an earlier one may still read it")
            self.pipe_last_start, self.pipe_last_done = start, done
            for r in reads:
                self.pipe_reads.setdefault(r, []).append(done)
            for w in writes:
                self.pipe_writes.setdefault(w, []).append(done)
            self.op_done.append(done)
        elif kind == "commit":
            done = max([self.t] + self.op_done) + 1
            self.seq += 1
            self.events.append((done, self.seq, lambda bar=act[1]: self._arrive(bar)))
        elif kind in ("read", "write"):
            self._access(role, kind, act[1])
        elif kind == "put":
            self._access(role, "write", act[1])
            self.values[act[1]] = act[2]
        elif kind == "get":
            self._access(role, "read", act[1])
            if self.values.get(act[1]) != act[2]:
                self.err(f"{role}: {act[1]} holds {self.values.get(act[1])}, expected {act[2]}")
        else:
            raise ValueError(f"unknown action {act!r}")

    # ------------------------------------------------------------------------------------------------ run
    def run(self, max_steps=3_000_000):
        st = {n: {"gen": g, "wait": None, "done": False, "sleep": 0} for n, g in self.roles.items()}
        for _ in range(max_steps):
            runnable, sleeping = [], False
            for n, s in st.items():
                if s["done"]:
                    continue
                if s["sleep"]:
                    s["sleep"] -= 1
                    sleeping = True
                    continue
                w = s["wait"]
                if w is None or self.bars[w[0]].completed % 2 != w[1] % 2:
                    runnable.append(n)
            if runnable:
                n = self.rng.choice(runnable)
                s = st[n]
                if self.rng.random() < self.stall_p:
                    s["sleep"] = self.rng.randint(1, self.stall_max)
                    continue
                if s["wait"] is not None:
                    bar, k = s["wait"]
                    if self.bars[bar].completed != k + 1:
                        self.err(f"{n}: wait on {bar} for phase {k} passed with {self.bars[bar].completed} completed")
                    s["wait"] = None
                try:
                    act = next(s["gen"])
                except StopIteration:
                    s["done"] = True
                    continue
                if act[0] == "wait":
                    s["wait"] = (act[1], act[2])
                else:
                    self._do(n, act)
                if self.rng.random() < 0.3:
                    self._advance()
                continue
            if self.events:
                self._advance(force=True)
                continue
            if sleeping:
                continue
            if not all(s["done"] for s in st.values()):
                self.err("deadlock: " + ", ".join(f"{n} waits {s['wait']}" for n, s in st.items() if not s["done"]))
            return
        self.err("step limit")
