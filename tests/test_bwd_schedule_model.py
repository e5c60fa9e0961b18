"""A model of the synchronization protocol of the persistent backward kernel
(`csrc/saf_bwd_tc.cu`), checked under random schedules.

Each role of the kernel (TMA producer, MMA issuer, key-row warps, dQ warps) is
written here as a generator that performs the same barrier operations, in the
same order and with the same phase parities, as the CUDA code; the tensor
pipe executes issued MMAs and commits in order, and TMA copies land at random
times.  mbarriers follow the hardware rule: a wait for parity p passes while
the barrier's phase count c has c % 2 != p.  For every run the model checks:

  * no deadlock (every role finishes for any interleaving tried);
  * no wait finds its barrier more than one phase past the completion it is
    waiting for (that would alias the parity and pass or block wrongly);
  * every read of a shared-memory stage or a TMEM region, by a thread or by
    an MMA when the pipe executes it, sees exactly the version written for its
    tile (catches both read-before-write and overwrite-before-read).

Items are random sequences of ordinary and replaced key blocks with 1 to 5
query-block tiles, as one CTA of the persistent grid meets them.
"""
import random

import pytest

NQS = 3  # Q/dO ring depth


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

    def __init__(self, rng):
        self.rng = rng
        self.bars = {}
        self.tag = {}          # resource -> version written last
        self.inflight = set()  # resources a TMA copy is writing
        self.pipe = []         # issued MMAs / commits not yet executed
        self.tma = []          # (barrier, bytes, resources) copies in flight
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

    def step_tma(self, i):
        bar, nbytes, resources = self.tma.pop(i)
        for res in resources:
            self.inflight.discard(res)
        self.bars[bar].complete_tx(nbytes)


# Roles.  A role yields ("wait", barrier, k, parity) to wait for completion k
# (0-based; k = -1: a fresh barrier, which the producer-side parity passes) and
# performs everything else directly on the machine between yields.

def W(name, k, parity):
    return ("wait", name, k, parity)


def producer(m, items):
    s = u = nk = 0
    G = 0
    for n, it in enumerate(items + [None]):
        yield W(f"ite{n & 1}", (n >> 1) - 1, ((n >> 1) & 1) ^ 1)
        m.slot[n & 1] = it
        m.bars[f"itf{n & 1}"].arrive()
        if it is None:
            return
        rep, ntiles = it
        if not rep:
            kb = nk & 1
            yield W(f"ke{kb}", (nk >> 1) - 1, ((nk >> 1) & 1) ^ 1)
            m.bars[f"kf{kb}"].expect_tx(1)
            m.write(f"K{kb}", ("K", nk), "producer")
            m.inflight.add(f"K{kb}")
            m.tma.append((f"kf{kb}", 1, [f"K{kb}"]))
        for t in range(ntiles):
            yield W(f"qe{s}", u - 1, (u & 1) ^ 1)
            res = [f"DO{s}", f"VEC1_{s}"] + ([] if rep else [f"Q{s}", f"VEC2_{s}"])
            for r in res:
                m.write(r, (r.rstrip("0123456789_"), G), "producer")
                m.inflight.add(r)
            m.bars[f"qf{s}"].expect_tx(len(res))
            m.tma.append((f"qf{s}", len(res), res))
            if not rep and t == 0:
                yield W("ve", nk - 1, (nk & 1) ^ 1)
                m.bars["vf"].expect_tx(1)
                m.write("V", ("V", nk), "producer")
                m.inflight.add("V")
                m.tma.append(("vf", 1, ["V"]))
            G += 1
            s += 1
            if s == NQS:
                s, u = 0, u + 1
        if not rep:
            nk += 1


def take(m, n):
    yield W(f"itf{n & 1}", n >> 1, (n >> 1) & 1)
    it = m.slot[n & 1]
    m.bars[f"ite{n & 1}"].arrive()
    return it


def mma_issuer(m):
    s = ph = 0
    go = gr = nk = 0
    G = 0
    n = 0
    while True:
        it = yield from take(m, n)
        if it is None:
            return
        rep, ntiles = it

        def mma(reads, writes, who):
            m.pipe.append(("mma", reads, writes, who))

        def commit(name):
            m.pipe.append(("commit", name))

        def ring(g):
            return g % NQS, (g // NQS) & 1, g // NQS

        if not rep:
            kb = nk & 1
            yield W(f"kf{kb}", nk >> 1, (nk >> 1) & 1)
            s0, p0, u0 = ring(G)
            assert (s0, p0) == (s, ph)
            yield W(f"qf{s0}", u0, p0)
            mma([(f"K{kb}", ("K", nk)), (f"Q{s0}", ("Q", G))], [("C_S", ("S", go))], "S")
            commit("s")
            yield W("vf", nk, nk & 1)
            mma([("V", ("V", nk)), (f"DO{s0}", ("DO", G))], [("C_DP", ("dP", go))], "dP")
            commit("dp")
            if ntiles == 1:
                commit("ve")
            for t in range(ntiles):
                g = G + t
                st, _, _ = ring(g)
                s1, p1, u1 = ring(g + 1)
                yield W("p", go, go & 1)
                if t == 0 and n > 0:
                    yield W("acr", n - 1, (n - 1) & 1)
                acc_in = [("C_DV", ("dV", n, t - 1))] if t > 0 else []
                mma([("C_S", ("P", go)), (f"DO{st}", ("DO", g))] + acc_in, [("C_DV", ("dV", n, t))], "dV")
                more = t + 1 < ntiles
                if more:
                    yield W(f"qf{s1}", u1, p1)
                    mma([(f"K{kb}", ("K", nk)), (f"Q{s1}", ("Q", g + 1))], [("C_S", ("S", go + 1))], "S")
                    commit("s")
                yield W("ds", go, go & 1)
                acc_in = [("C_DK", ("dK", n, t - 1))] if t > 0 else []
                mma([("C_DP", ("dS", go)), (f"Q{st}", ("Q", g))] + acc_in, [("C_DK", ("dK", n, t))], "dK")
                b = go & 1
                yield W(f"dqe{b}", (go >> 1) - 1, ((go >> 1) & 1) ^ 1)
                mma([("DS", ("dS", go)), (f"K{kb}", ("K", nk))], [(f"C_DQ{b}", ("dQ", go))], "dQ")
                commit(f"dqf{b}")
                if more:
                    mma([("V", ("V", nk)), (f"DO{s1}", ("DO", g + 1))], [("C_DP", ("dP", go + 1))], "dP")
                    commit("dp")
                    if t + 2 == ntiles:
                        commit("ve")
                commit(f"qe{st}")
                go += 1
            commit("acc")
            commit(f"ke{kb}")
            nk += 1
        else:
            for t in range(ntiles):
                g = G + t
                st, pt, ut = ring(g)
                yield W(f"qf{st}", ut, pt)
                yield W(f"pb{gr & 1}", gr >> 1, (gr >> 1) & 1)
                if t == 0 and n > 0:
                    yield W("acr", n - 1, (n - 1) & 1)
                wreg = "C_S" if gr % 2 == 0 else "C_DP"
                acc_in = [("C_DV", ("dV", n, t - 1))] if t > 0 else []
                mma([(wreg, ("W", gr)), (f"DO{st}", ("DO", g))] + acc_in, [("C_DV", ("dV", n, t))], "dV(W)")
                commit(f"wb{gr & 1}")
                commit(f"qe{st}")
                gr += 1
            commit("acc")
        G += ntiles
        s, ph = G % NQS, (G // NQS) & 1
        n += 1


def key_rows(m):
    s = u = 0
    go = gr = 0
    G = 0
    n = 0
    while True:
        it = yield from take(m, n)
        if it is None:
            return
        rep, ntiles = it
        for t in range(ntiles):
            g = G + t
            yield W(f"qf{s}", u, u & 1)
            if not rep:
                yield W("s", go, go & 1)
                m.read("C_S", ("S", go), "rows P")
                m.read(f"VEC1_{s}", ("VEC", g), "rows P")
                m.write("C_S", ("P", go), "rows P")
                m.bars["p"].arrive()
                yield W("dp", go, go & 1)
                m.read("C_DP", ("dP", go), "rows dS")
                m.read(f"VEC2_{s}", ("VEC", g), "rows dS")
                m.write("C_DP", ("dS", go), "rows dS")
                m.write("DS", ("dS", go), "rows dS")
                m.bars["ds"].arrive()
                go += 1
            else:
                if gr >= 2:
                    yield W(f"wb{gr & 1}", (gr >> 1) - 1, ((gr >> 1) & 1) ^ 1)
                m.read(f"VEC1_{s}", ("VEC", g), "rows W")
                m.write("C_S" if gr % 2 == 0 else "C_DP", ("W", gr), "rows W")
                m.bars[f"pb{gr & 1}"].arrive()
                gr += 1
            s += 1
            if s == NQS:
                s, u = 0, u + 1
        G += ntiles
        yield W("acc", n, n & 1)
        m.read("C_DV", ("dV", n, ntiles - 1), "rows epilogue")
        if not rep:
            m.read("C_DK", ("dK", n, ntiles - 1), "rows epilogue")
        m.bars["acr"].arrive()
        n += 1


def dq_warps(m):
    go = 0
    n = 0
    while True:
        it = yield from take(m, n)
        if it is None:
            return
        rep, ntiles = it
        n += 1
        if rep:
            continue
        for _ in range(ntiles):
            b = go & 1
            yield W(f"dqf{b}", go >> 1, (go >> 1) & 1)
            m.read(f"C_DQ{b}", ("dQ", go), "dQ warps")
            m.bars[f"dqe{b}"].arrive()
            go += 1


def run(items, seed):
    rng = random.Random(seed)
    m = Machine(rng)
    for b in range(2):
        m.bar(f"itf{b}")
        m.bar(f"ite{b}", 3)  # MMA issuer, key rows, dQ warps
        for name in ("kf", "ke", "dqf", "dqe", "wb", "pb"):
            m.bar(f"{name}{b}")
    for st in range(NQS):
        m.bar(f"qf{st}")
        m.bar(f"qe{st}")
    for name in ("vf", "ve", "s", "dp", "p", "ds", "acc", "acr"):
        m.bar(name)
    roles = {"producer": producer(m, items), "mma": mma_issuer(m), "rows": key_rows(m), "dq": dq_warps(m)}
    waiting = {}
    for name, gen in roles.items():
        waiting[name] = next(gen, None)
    # each actor gets its own speed for the run (log-uniform over three decades),
    # so schedules where one role lags far behind the others come up often
    speed = {name: 10 ** rng.uniform(-3, 0) for name in list(roles) + ["pipe", "tma"]}
    checked = set()
    steps = 0
    while True:
        steps += 1
        if steps > 200000:
            raise ModelError("no progress")
        ready = []
        for name, w in waiting.items():
            if w is None:
                continue
            _, bname, k, parity = w
            bar = m.bars[bname]
            key = (name, bname, k)
            if key not in checked:
                checked.add(key)
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
        for i in range(len(m.tma)):
            ready.append(("tma", i))
        if not ready:
            if all(w is None for w in waiting.values()):
                return steps
            stuck = {k: v[1:] for k, v in waiting.items() if v is not None}
            raise ModelError(f"deadlock: {stuck}")
        weights = [speed[arg] if kind == "role" else speed[kind] for kind, arg in ready]
        kind, arg = rng.choices(ready, weights)[0]
        if kind == "pipe":
            m.step_pipe()
        elif kind == "tma":
            m.step_tma(arg)
        else:
            waiting[arg] = next(roles[arg], None)


def random_items(rng):
    return [(rng.random() < 0.35, rng.randint(1, 5)) for _ in range(rng.randint(1, 7))]


def test_tag_naming_is_consistent():
    """The producer versions a stage by its name without the stage index
    ("VEC1_2" and "VEC2_2" -> "VEC", "Q2" -> "Q"), which the readers expect."""
    assert "VEC1_2".rstrip("0123456789_") == "VEC"
    assert "Q2".rstrip("0123456789_") == "Q" and "DO0".rstrip("0123456789_") == "DO"


@pytest.mark.parametrize("seed", range(40))
def test_random_item_sequences_and_schedules(seed):
    rng = random.Random(1000 + seed)
    items = random_items(rng)
    for sched in range(25):
        run(items, seed * 100 + sched)


def test_edge_sequences():
    """Single-tile items (the last dP^T is the first), kinds alternating, long runs of one kind."""
    cases = [
        [(False, 1)] * 6,
        [(True, 1)] * 6,
        [(False, 1), (True, 1)] * 4,
        [(True, 3), (False, 1), (True, 2), (False, 4), (False, 1)],
        [(False, 5), (False, 5), (False, 5)],
        [(True, 5), (True, 4), (False, 2), (True, 1)],
    ]
    for i, items in enumerate(cases):
        for sched in range(40):
            run(items, 7000 + 100 * i + sched)


def _mutant(monkeypatch, fn_name, transform):
    import tests.test_bwd_schedule_model as mod
    import inspect
    src = inspect.getsource(getattr(mod, fn_name))
    new = transform(src)
    assert new != src
    ns = {}
    exec(compile(new, "<mutant>", "exec"), mod.__dict__, ns)
    monkeypatch.setattr(mod, fn_name, ns[fn_name])


@pytest.mark.parametrize("fn_name,old,new", [
    # K reloaded into a stage whose item's MMAs still read it
    ("producer", 'yield W(f"ke{kb}", (nk >> 1) - 1, ((nk >> 1) & 1) ^ 1)', 'pass'),
    # a Q/dO ring stage refilled before its tile's MMAs are done
    ("producer", 'yield W(f"qe{s}", u - 1, (u & 1) ^ 1)', 'pass'),
    # V reloaded before the previous item's last dP^T has read it
    ("producer", 'yield W("ve", nk - 1, (nk & 1) ^ 1)', 'pass'),
    # a replaced head's W buffer rewritten before its MMA ran
    ("key_rows", "if gr >= 2:\n", "if False:\n"),
    # the dQ TMEM buffer reused without waiting for the dQ warps
    ("mma_issuer", 'yield W(f"dqe{b}", (go >> 1) - 1, ((go >> 1) & 1) ^ 1)', 'pass'),
    # the rows read dP^T before its MMA has run
    ("key_rows", 'yield W("dp", go, go & 1)', 'pass'),
], ids=["no_ke", "no_qe", "no_ve", "no_wb", "no_dqe", "no_dp_wait"])
def test_model_catches_planted_mistakes(monkeypatch, fn_name, old, new):
    """Each planted mistake in the protocol is caught on some schedule."""
    _mutant(monkeypatch, fn_name, lambda src: src.replace(old, new))
    import tests.test_bwd_schedule_model as mod
    rng = random.Random(5)
    caught = False
    for trial in range(300):
        items = [(rng.random() < 0.35, rng.randint(1, 4)) for _ in range(rng.randint(2, 6))]
        try:
            mod.run(items, trial)
        except ModelError:
            caught = True
            break
    assert caught


def test_readout_barrier_is_implied_by_row_order(monkeypatch):
    """The MMA warp's wait for the dK/dV read-out before an item's first dV is
    implied: the same row warps read dK/dV out before they produce the next
    item's first P^T (or W), which that dV waits for.  Without the wait the
    protocol stays correct on every schedule tried."""
    _mutant(monkeypatch, "mma_issuer",
            lambda src: src.replace('if t == 0 and n > 0:\n                    yield W("acr"',
                                    'if False:\n                    yield W("acr"'))
    import tests.test_bwd_schedule_model as mod
    rng = random.Random(9)
    for trial in range(300):
        items = [(rng.random() < 0.35, rng.randint(1, 4)) for _ in range(rng.randint(2, 6))]
        mod.run(items, trial)
