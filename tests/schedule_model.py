"""Machinery for checking the persistent kernels' synchronization protocols on
the CPU: mbarriers with the hardware's phase-parity rule, versioned resources
(shared-memory stages, TMEM regions), an in-order tensor pipe, TMA copies that
land at random times, and a scheduler that interleaves the roles at random.

A role is a generator.  It yields ("wait", barrier, k, parity) to wait for
completion k of a barrier (0-based; k = -1 for the first use of a "free"
barrier, which the producer-side parity passes at once) with the parity the
kernel passes to try_wait, and does everything else directly on the machine
between yields.  The scheduler checks, at each wait, that the kernel's parity
is the one completion k needs and that the barrier is not already a phase
past it (the parity would alias); reads check the version of what they read.
"""
import inspect


class ModelError(AssertionError):
    pass


class Barrier:
    def __init__(self, name, count):
        self.name, self.count = name, count
        self.pending, self.tx, self.phases = count, 0, 0

    def _maybe_complete(self):
        if self.pending == 0 and self.tx == 0:
            self.phases += 1
            self.pending = self.count

    def arrive(self):
        if self.pending <= 0:
            raise ModelError(f"{self.name}: arrival beyond the expected count")
        self.pending -= 1
        self._maybe_complete()

    def expect_tx(self, nbytes):  # arrive.expect_tx: one arrival plus a transaction count
        self.tx += nbytes
        self.arrive()

    def complete_tx(self, nbytes):
        self.tx -= nbytes
        if self.tx < 0:
            raise ModelError(f"{self.name}: more bytes than expected")
        self._maybe_complete()


class Machine:
    """Barriers, versioned resources, the in-order tensor pipe and the TMA engine."""

    def __init__(self):
        self.bars = {}
        self.tag = {}          # resource -> version written last
        self.inflight = set()  # resources a TMA copy is writing
        self.pipe = []         # issued MMAs / commits not yet executed
        self.tma = []          # (barrier, units, resources) copies in flight
        self.stores = []       # (issuer key, resource, version, who, number) stores in flight
        self.store_seq = {}    # issuer key -> stores made
        self.store_done = {}   # issuer key -> numbers of the stores that have read their source
        self.slot = [None, None]

    def bar(self, name, count=1):
        if name not in self.bars:
            self.bars[name] = Barrier(name, count)
        return self.bars[name]

    def read(self, res, want, who):
        if res in self.inflight:
            raise ModelError(f"{who} reads {res} while a copy into it is in flight")
        if self.tag.get(res) != want:
            raise ModelError(f"{who} reads {res}: has {self.tag.get(res)}, wants {want}")

    def write(self, res, version, who):
        if res in self.inflight:
            raise ModelError(f"{who} writes {res} while a copy into it is in flight")
        self.tag[res] = version

    def copy(self, bar, writes, who):
        """A TMA copy: the barrier expects it (one arrival plus its size); the
        destinations carry the new versions and count as in flight until it lands."""
        for res, version in writes:
            self.write(res, version, who)
            self.inflight.add(res)
        self.bars[bar].expect_tx(len(writes))
        self.tma.append((bar, len(writes), [res for res, _ in writes]))

    def mma(self, reads, writes, who):
        self.pipe.append(("mma", reads, writes, who))

    def commit(self, bar):
        self.pipe.append(("commit", bar))

    def step_pipe(self):
        op = self.pipe.pop(0)
        if op[0] == "mma":
            _, reads, writes, who = op
            for res, want in reads:
                self.read(res, want, who)
            for res, version in writes:
                self.write(res, version, who)
        else:
            self.bars[op[1]].arrive()

    def store(self, bar, res, want, who):
        """A bulk store out of shared memory: reads `res` (which must still hold
        `want`) whenever it runs, in any order with the issuer's other stores;
        `bar` names the issuer's stores for its bulk-group waits (WC)."""
        seq = self.store_seq.get(bar, 0)
        self.store_seq[bar] = seq + 1
        self.stores.append((bar, res, want, who, seq))

    def step_store(self, i):
        bar, res, want, who, seq = self.stores.pop(i)
        self.read(res, want, who)
        self.store_done.setdefault(bar, set()).add(seq)

    def stores_done_below(self, bar, upto):
        done = self.store_done.get(bar, set())
        return all(q in done for q in range(upto))

    def step_tma(self, i):
        bar, units, resources = self.tma.pop(i)
        for res in resources:
            self.inflight.discard(res)
        self.bars[bar].complete_tx(units)


def W(name, k, parity):
    return ("wait", name, k, parity)


def WC(name, upto):
    """A bulk-group wait: until every store the issuer made through `name`
    before its store number `upto` (counted from 0) has read its source, the
    later ones may still be pending (cp.async.bulk.wait_group.read N leaves
    the N most recent groups pending).  No phase parity is involved."""
    return ("count", name, upto, None)


def take(m, n):
    """A consumer takes work item n from the two-slot ring (-1 / None: done)."""
    yield W(f"itf{n & 1}", n >> 1, (n >> 1) & 1)
    it = m.slot[n & 1]
    m.bars[f"ite{n & 1}"].arrive()
    return it


def publish(m, n, item):
    """The producer publishes item n once the slot's previous item was taken."""
    yield W(f"ite{n & 1}", (n >> 1) - 1, ((n >> 1) & 1) ^ 1)
    m.slot[n & 1] = item
    m.bars[f"itf{n & 1}"].arrive()


def simulate(m, roles, rng, max_steps=200000):
    """Interleaves the roles, the pipe and the copies at random until all roles
    finish; raises ModelError on a deadlock or a protocol violation.  Each
    actor gets its own speed for the run (log-uniform over three decades), so
    schedules where one role lags far behind the others come up often."""
    waiting = {name: next(gen, None) for name, gen in roles.items()}
    speed = {name: 10 ** rng.uniform(-3, 0) for name in list(roles) + ["pipe", "tma"]}
    checked = set()
    for _ in range(max_steps):
        ready = []
        for name, w in waiting.items():
            if w is None:
                continue
            kind, bname, k, parity = w
            if kind == "count":
                if m.stores_done_below(bname, k):
                    ready.append(("role", name))
                continue
            bar = m.bars[bname]
            if (name, bname, k) not in checked:
                checked.add((name, bname, k))
                if k >= 0 and parity != (k & 1):
                    raise ModelError(f"{name}: parity {parity} for completion {k} of {bname}")
                if bar.phases > k + 1:
                    raise ModelError(f"{name}: {bname} is {bar.phases - k - 1} phases past completion {k}")
            if bar.phases % 2 != parity:
                if bar.phases < k + 1:
                    raise ModelError(f"{name}: wait on {bname} passes before completion {k}")
                ready.append(("role", name))
        if m.pipe:
            ready.append(("pipe", None))
        ready += [("tma", i) for i in range(len(m.tma))]
        ready += [("store", i) for i in range(len(m.stores))]
        if not ready:
            if all(w is None for w in waiting.values()):
                return
            stuck = {k: v[1:] for k, v in waiting.items() if v is not None}
            raise ModelError(f"deadlock: {stuck}")
        weights = [speed[arg] if kind == "role" else speed["tma" if kind == "store" else kind] for kind, arg in ready]
        kind, arg = rng.choices(ready, weights)[0]
        if kind == "pipe":
            m.step_pipe()
        elif kind == "tma":
            m.step_tma(arg)
        elif kind == "store":
            m.step_store(arg)
        else:
            waiting[arg] = next(roles[arg], None)
    raise ModelError("no progress")


def mutate(monkeypatch, module, fn_name, old, new):
    """Replaces `old` by `new` in the source of module.fn_name (a planted mistake)."""
    src = inspect.getsource(getattr(module, fn_name))
    changed = src.replace(old, new)
    assert changed != src, f"{old!r} not found in {fn_name}"
    ns = {}
    exec(compile(changed, "<mutant>", "exec"), module.__dict__, ns)
    monkeypatch.setattr(module, fn_name, ns[fn_name])
