"""A model of the synchronization protocol of the persistent backward kernel
(`csrc/saf_bwd_tc.cu`), checked under random schedules.

Each role of the kernel (TMA producer, MMA issuer, each of the 8 key-row warps
and each of the 4 dQ warps, with the kernel's arrival counts and their own
slices of the TMEM regions) is written here as a generator that performs the same barrier operations, in the
same order and with the same phase parities, as the CUDA code (the machinery
is in tests/schedule_model.py).  For every run the model checks:

  * no deadlock (every role finishes for the interleaving tried);
  * no wait finds its barrier a phase past the completion it waits for (that
    would alias the parity);
  * every read of a shared-memory stage or a TMEM region, by a thread or by
    an MMA when the pipe executes it, sees exactly the version written for its
    tile (catches both read-before-write and overwrite-before-read).

Items are random sequences of ordinary and replaced key blocks with 1 to 5
query-block tiles, as one CTA of the persistent grid meets them.
"""
import random

import pytest

from tests.schedule_model import Machine, ModelError, W, WC, mutate, publish, simulate, take

NQS = 3  # Q/dO ring depth
# dK, dV are declared complete (bar_acc) after the item's last dQ MMA, the
# last reader of the dS^T area that the row warps then stage dK/dV rows in
# (the alternative, right after the last dK MMA, is the planted mistake below)
ACC_AFTER_DQ = True
ROWS = 8  # key-row warps: each owns one slice (lane quarter x column half) of S^T, dP^T and dS^T
DQW = 4   # dQ warps: each owns one lane quarter of the dQ tiles


def parts(res, n):
    """The per-warp slices of a region that the MMA reads or writes whole."""
    return [f"{res}.{w}" for w in range(n)]


def all_of(res, n, version):
    return [(r, version) for r in parts(res, n)]


def ring(g):
    """Stage, phase parity and pass of the g-th query block of the ring."""
    return g % NQS, (g // NQS) & 1, g // NQS


def producer(m, items):
    nk = 0  # ordinary items so far
    G = 0   # query blocks so far (ring position)
    for n, it in enumerate(items + [None]):
        yield from publish(m, n, it)
        if it is None:
            return
        rep, ntiles = it
        if not rep:
            kb = nk & 1
            yield W(f"ke{kb}", (nk >> 1) - 1, ((nk >> 1) & 1) ^ 1)
            m.copy(f"kf{kb}", [(f"K{kb}", ("K", nk))], "producer")
        for t in range(ntiles):
            s, _, u = ring(G)
            yield W(f"qe{s}", u - 1, (u & 1) ^ 1)
            res = [(f"DO{s}", ("DO", G)), (f"VEC1_{s}", ("VEC", G))]
            if not rep:
                res += [(f"Q{s}", ("Q", G)), (f"VEC2_{s}", ("VEC", G))]
            m.copy(f"qf{s}", res, "producer")
            if not rep and t == 0:
                yield W("ve", nk - 1, (nk & 1) ^ 1)
                m.copy("vf", [("V", ("V", nk))], "producer")
            G += 1
        if not rep:
            nk += 1


def mma_issuer(m):
    go = gr = nk = 0  # ordinary tiles, replaced tiles, ordinary items so far
    G = 0
    n = 0
    while True:
        it = yield from take(m, n)
        if it is None:
            return
        rep, ntiles = it
        if not rep:
            kb = nk & 1
            yield W(f"kf{kb}", nk >> 1, (nk >> 1) & 1)
            s0, p0, u0 = ring(G)
            yield W(f"qf{s0}", u0, p0)
            m.mma([(f"K{kb}", ("K", nk)), (f"Q{s0}", ("Q", G))], all_of("C_S", ROWS, ("S", go)), "S")
            m.commit("s")
            yield W("vf", nk, nk & 1)
            m.mma([("V", ("V", nk)), (f"DO{s0}", ("DO", G))], all_of("C_DP", ROWS, ("dP", go)), "dP")
            m.commit("dp")
            if ntiles == 1:
                m.commit("ve")
            for t in range(ntiles):
                g = G + t
                st, _, _ = ring(g)
                s1, p1, u1 = ring(g + 1)
                yield W("p", go, go & 1)
                if t == 0 and n > 0:
                    yield W("acr", n - 1, (n - 1) & 1)
                acc_in = [("C_DV", ("dV", n, t - 1))] if t > 0 else []
                m.mma(all_of("C_S", ROWS, ("P", go)) + [(f"DO{st}", ("DO", g))] + acc_in, [("C_DV", ("dV", n, t))], "dV")
                more = t + 1 < ntiles
                if more:
                    yield W(f"qf{s1}", u1, p1)
                    m.mma([(f"K{kb}", ("K", nk)), (f"Q{s1}", ("Q", g + 1))], all_of("C_S", ROWS, ("S", go + 1)), "S")
                    m.commit("s")
                yield W("ds", go, go & 1)
                acc_in = [("C_DK", ("dK", n, t - 1))] if t > 0 else []
                m.mma(all_of("C_DP", ROWS, ("dS", go)) + [(f"Q{st}", ("Q", g))] + acc_in, [("C_DK", ("dK", n, t))], "dK")
                if not more and not ACC_AFTER_DQ:
                    m.commit("acc")
                b = go & 1
                yield W(f"dqe{b}", (go >> 1) - 1, ((go >> 1) & 1) ^ 1)
                m.mma(all_of("DS", ROWS, ("dS", go)) + [(f"K{kb}", ("K", nk))], all_of(f"C_DQ{b}", DQW, ("dQ", go)), "dQ")
                m.commit(f"dqf{b}")
                if not more and ACC_AFTER_DQ:
                    m.commit("acc")
                if more:
                    m.mma([("V", ("V", nk)), (f"DO{s1}", ("DO", g + 1))], all_of("C_DP", ROWS, ("dP", go + 1)), "dP")
                    m.commit("dp")
                    if t + 2 == ntiles:
                        m.commit("ve")
                m.commit(f"qe{st}")
                go += 1
            m.commit(f"ke{kb}")
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
                m.mma(all_of(wreg, ROWS, ("W", gr)) + [(f"DO{st}", ("DO", g))] + acc_in, [("C_DV", ("dV", n, t))], "dV(W)")
                m.commit(f"wb{gr & 1}")
                m.commit(f"qe{st}")
                gr += 1
            m.commit("acc")
        G += ntiles
        n += 1


def key_rows(m, w):
    go = gr = 0
    G = 0
    n = 0
    ns = 0  # dK/dV boxes this warp has stored from its slice of the dS^T area
    while True:
        it = yield from take(m, n)
        if it is None:
            return
        rep, ntiles = it
        for t in range(ntiles):
            g = G + t
            s, p, u = ring(g)
            yield W(f"qf{s}", u, p)
            if not rep:
                yield W("s", go, go & 1)
                m.read(f"C_S.{w}", ("S", go), "rows P")
                m.read(f"VEC1_{s}", ("VEC", g), "rows P")
                m.write(f"C_S.{w}", ("P", go), "rows P")
                m.bars["p"].arrive()
                yield W("dp", go, go & 1)
                m.read(f"C_DP.{w}", ("dP", go), "rows dS")
                m.read(f"VEC2_{s}", ("VEC", g), "rows dS")
                if t == 0 and ns > 0:  # the last box has been read out of DS.w
                    yield WC(f"sr{w}", ns)
                m.write(f"C_DP.{w}", ("dS", go), "rows dS")
                m.write(f"DS.{w}", ("dS", go), "rows dS")
                m.bars["ds"].arrive()
                go += 1
            else:
                if gr >= 2:
                    yield W(f"wb{gr & 1}", (gr >> 1) - 1, ((gr >> 1) & 1) ^ 1)
                m.read(f"VEC1_{s}", ("VEC", g), "rows W")
                m.write(f"{'C_S' if gr % 2 == 0 else 'C_DP'}.{w}", ("W", gr), "rows W")
                m.bars[f"pb{gr & 1}"].arrive()
                gr += 1
        G += ntiles
        # read-out of dK, dV (a replaced head's dK columns are not read: its rows are zeros)
        yield W("acc", n, n & 1)
        m.read("C_DV", ("dV", n, ntiles - 1), "rows epilogue")
        if not rep:
            m.read("C_DK", ("dK", n, ntiles - 1), "rows epilogue")
        m.bars["acr"].arrive()
        # the warp's dK or dV rows staged in its slice of the dS^T area, then
        # stored out by one bulk store (after the previous one has read it)
        if ns > 0:
            yield WC(f"sr{w}", ns)
        m.write(f"DS.{w}", ("stage", n), "rows stage")
        m.store(f"sr{w}", f"DS.{w}", ("stage", n), "dK/dV store")
        ns += 1
        n += 1


def dq_warp(m, w):
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
            m.read(f"C_DQ{b}.{w}", ("dQ", go), "dQ warps")
            m.bars[f"dqe{b}"].arrive()
            go += 1


def run(items, seed):
    m = Machine()
    for b in range(2):
        m.bar(f"itf{b}")
        m.bar(f"ite{b}", 1 + ROWS + DQW)  # each consumer warp acknowledges an item
        for name in ("kf", "ke", "dqf", "wb"):
            m.bar(f"{name}{b}")
        m.bar(f"dqe{b}", DQW)
        m.bar(f"pb{b}", ROWS)
    for st in range(NQS):
        m.bar(f"qf{st}")
        m.bar(f"qe{st}")
    for name in ("vf", "ve", "s", "dp", "acc"):
        m.bar(name)
    for name in ("p", "ds", "acr"):
        m.bar(name, ROWS)
    roles = {"producer": producer(m, items), "mma": mma_issuer(m)}
    roles.update({f"rows{w}": key_rows(m, w) for w in range(ROWS)})
    roles.update({f"dq{w}": dq_warp(m, w) for w in range(DQW)})
    simulate(m, roles, random.Random(seed))


def random_items(rng, max_tiles=5):
    return [(rng.random() < 0.35, rng.randint(1, max_tiles)) for _ in range(rng.randint(1, 7))]


@pytest.mark.parametrize("seed", range(40))
def test_random_item_sequences_and_schedules(seed):
    rng = random.Random(1000 + seed)
    items = random_items(rng)
    for sched in range(10):
        run(items, seed * 100 + sched)


def test_edge_sequences():
    """Single-tile items (an item's first dP^T is its last), kinds alternating,
    long runs of one kind."""
    cases = [
        [(False, 1)] * 6,
        [(True, 1)] * 6,
        [(False, 1), (True, 1)] * 4,
        [(True, 3), (False, 1), (True, 2), (False, 4), (False, 1)],
        [(False, 5), (False, 5), (False, 5)],
        [(True, 5), (True, 4), (False, 2), (True, 1)],
    ]
    for i, items in enumerate(cases):
        for sched in range(20):
            run(items, 7000 + 100 * i + sched)


def _caught(seed):
    import tests.test_bwd_schedule_model as mod
    rng = random.Random(seed)
    for trial in range(300):
        try:
            mod.run(random_items(rng, 4), trial)
        except ModelError:
            return True
    return False


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
    # dS^T written over a dK/dV box its store has not read yet
    ("key_rows", "if t == 0 and ns > 0:", "if False:"),
    # a box staged over the previous box before its store has read it
    ("key_rows", "if ns > 0:\n", "if False:\n"),
], ids=["no_ke", "no_qe", "no_ve", "no_wb", "no_dqe", "no_dp_wait", "no_store_read_ds", "no_store_read_stage"])
def test_model_catches_planted_mistakes(monkeypatch, fn_name, old, new):
    """Each planted mistake in the protocol is caught on some schedule."""
    import tests.test_bwd_schedule_model as mod
    mutate(monkeypatch, mod, fn_name, old, new)
    assert _caught(5)


def test_acc_before_last_dq_is_caught(monkeypatch):
    """dK, dV declared complete right after the item's last dK MMA: the rows
    stage their dK/dV rows over dS^T that the last dQ MMA has not read yet."""
    import tests.test_bwd_schedule_model as mod
    monkeypatch.setattr(mod, "ACC_AFTER_DQ", False)
    assert _caught(5)


def test_readout_barrier_is_implied_by_row_order(monkeypatch):
    """The MMA warp's wait for the dK/dV read-out before an item's first dV is
    implied: the same row warps read dK/dV out before they produce the next
    item's first P^T (or W), which that dV waits for.  Without the wait the
    protocol stays correct on every schedule tried."""
    import tests.test_bwd_schedule_model as mod
    mutate(monkeypatch, mod, "mma_issuer", 'if t == 0 and n > 0:\n                    yield W("acr"',
           'if False:\n                    yield W("acr"')
    assert not _caught(9)
