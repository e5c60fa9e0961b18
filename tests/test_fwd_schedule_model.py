"""A model of the synchronization protocol of the persistent forward kernel
(`csrc/saf_fwd_tc.cu`), checked under random schedules.

The roles (TMA producer, MMA issuer, each of the 4 query-row warps with the
kernel's arrival counts and its own lane quarter of S, P and O) perform the kernel's
barrier operations in its order and with its phase parities (machinery in
tests/schedule_model.py).  Resources: Q in two buffers (this item, the next),
K and V rings of two stages each (K loaded one block ahead of V), the S
columns of TMEM (two 64-column halves, which a replaced head uses as its two
W buffers), P and O.  Checked on every run: no deadlock, no parity aliasing,
and every read sees the version written for its block.  The row warps' lazy
O rescale is modelled as always happening (a superset of the real accesses).
"""
import random

import pytest

from tests.schedule_model import Machine, ModelError, W, WC, mutate, publish, simulate, take

NSK = NSV = 2  # K, V ring stages
ROWS = 4       # query-row warps: each owns one lane quarter of S, P and O


def all_of(res, version):
    """A region the MMA reads or writes whole: every warp's slice."""
    return [(f"{res}.{w}", version) for w in range(ROWS)]


def producer(m, items):
    gk = gv = gr = nq = 0  # K, V, replaced blocks; ordinary items so far
    for n, it in enumerate(items + [None]):
        yield from publish(m, n, it)
        if it is None:
            return
        rep, nkb = it
        if not rep:
            b = nq & 1
            yield W(f"qe{b}", (nq >> 1) - 1, ((nq >> 1) & 1) ^ 1)
            m.copy(f"qf{b}", [(f"Q{b}", ("Q", nq))], "producer")
            nq += 1

        def load_k(j):
            g = gk + j
            s, u = g % NSK, g // NSK
            yield W(f"ke{s}", u - 1, (u & 1) ^ 1)
            m.copy(f"kf{s}", [(f"K{s}", ("K", g))], "producer")

        if not rep:
            yield from load_k(0)
        for j in range(nkb):
            if not rep and j + 1 < nkb:
                yield from load_k(j + 1)
            if rep:
                # a replaced block's W inputs (E and c) into stage gw & 1, once
                # the rows have built block gw - 2 from it
                gw = gr + j
                if gw >= 2:
                    yield W(f"pb{gw & 1}", (gw >> 1) - 1, ((gw >> 1) & 1) ^ 1)
                m.copy(f"wf{gw & 1}", [(f"WST{gw & 1}", ("WIN", gw))], "producer")
            g = gv + j
            s, u = g % NSV, g // NSV
            yield W(f"ve{s}", u - 1, (u & 1) ^ 1)
            m.copy(f"vf{s}", [(f"V{s}", ("V", g))], "producer")
        if rep:
            gr += nkb
        else:
            gk += nkb
        gv += nkb


def mma_issuer(m):
    gk = gv = go = gr = nq = 0
    n = 0
    while True:
        it = yield from take(m, n)
        if it is None:
            return
        rep, nkb = it
        b = nq & 1

        def issue_s(j):
            g = gk + j
            s, u = g % NSK, g // NSK
            yield W(f"kf{s}", u, u & 1)
            m.mma([(f"Q{b}", ("Q", nq)), (f"K{s}", ("K", g))],
                  all_of("S_lo", ("S", go + j)) + all_of("S_hi", ("S", go + j)), "S")
            m.commit("s")
            m.commit(f"ke{s}")
            if j == nkb - 1:
                m.commit(f"qe{b}")

        if not rep:
            yield W(f"qf{b}", nq >> 1, (nq >> 1) & 1)
            yield from issue_s(0)
        for j in range(nkb):
            if not rep and j + 1 < nkb:
                yield W("sf", go + j, (go + j) & 1)
                yield from issue_s(j + 1)
            g = gv + j
            s, u = g % NSV, g // NSV
            yield W(f"vf{s}", u, u & 1)
            wb = (gr + j) & 1
            if rep:
                yield W(f"pb{wb}", (gr + j) >> 1, ((gr + j) >> 1) & 1)
                a = all_of("S_lo" if wb == 0 else "S_hi", ("W", gr + j))
            else:
                yield W("p", go + j, (go + j) & 1)
                a = all_of("P", ("P", go + j))
            acc_in = all_of("O", ("O", n, j - 1)) if j > 0 else []
            m.mma(a + [(f"V{s}", ("V", g))] + acc_in, all_of("O", ("O", n, j)), "P.V")
            m.commit(f"ob{wb}" if rep else "o")
            m.commit(f"ve{s}")
        if rep:
            gr += nkb
        else:
            gk += nkb
            go += nkb
            nq += 1
        gv += nkb
        n += 1


def query_rows(m, w):
    go = gr = 0
    n = 0
    ns = 0  # O boxes this warp has stored from its staging area
    while True:
        it = yield from take(m, n)
        if it is None:
            return
        rep, nkb = it
        for j in range(nkb):
            if not rep:
                last = j == nkb - 1
                yield W("s", go + j, (go + j) & 1)
                m.read(f"S_lo.{w}", ("S", go + j), "rows")
                m.read(f"S_hi.{w}", ("S", go + j), "rows")
                if not last:
                    m.bars["sf"].arrive()
                if j > 0:
                    yield W("o", go + j - 1, (go + j - 1) & 1)
                    m.read(f"O.{w}", ("O", n, j - 1), "rows rescale")
                    m.write(f"O.{w}", ("O", n, j - 1), "rows rescale")
                if last:
                    # the diagonal block reads S a second time (its exp pass)
                    # and releases it only then
                    m.read(f"S_lo.{w}", ("S", go + j), "rows diagonal")
                    m.read(f"S_hi.{w}", ("S", go + j), "rows diagonal")
                m.write(f"P.{w}", ("P", go + j), "rows")
                if last:
                    m.bars["sf"].arrive()
                m.bars["p"].arrive()
            else:
                g = gr + j
                if g >= 2:
                    yield W(f"ob{g & 1}", (g >> 1) - 1, ((g >> 1) & 1) ^ 1)
                yield W(f"wf{g & 1}", g >> 1, (g >> 1) & 1)
                m.read(f"WST{g & 1}", ("WIN", g), "rows W")
                m.write(f"{'S_lo' if g % 2 == 0 else 'S_hi'}.{w}", ("W", g), "rows W")
                m.bars[f"pb{g & 1}"].arrive()
        gl = (gr if rep else go) + nkb - 1  # the item's last P.V
        if rep:
            yield W(f"ob{gl & 1}", gl >> 1, (gl >> 1) & 1)
        else:
            yield W("o", gl, gl & 1)
        m.read(f"O.{w}", ("O", n, nkb - 1), "rows epilogue")
        # two 32-column boxes through the warp's staging area, each written
        # once every earlier store has read it (a bulk-group wait for all)
        for c in range(2):
            if ns > 0:
                yield WC(f"sr{w}", ns)
            m.write(f"OST.{w}", ("O box", n, c), "rows stage")
            m.store(f"sr{w}", f"OST.{w}", ("O box", n, c), "O store")
            ns += 1
        if rep:
            gr += nkb
        else:
            go += nkb
        n += 1


def run(items, seed):
    m = Machine()
    for b in range(2):
        m.bar(f"itf{b}")
        m.bar(f"ite{b}", 1 + ROWS)  # the MMA warp and each row warp acknowledge an item
        for name in ("qf", "qe", "ob", "wf"):
            m.bar(f"{name}{b}")
        m.bar(f"pb{b}", ROWS)
    for s in range(NSK):
        m.bar(f"kf{s}")
        m.bar(f"ke{s}")
    for s in range(NSV):
        m.bar(f"vf{s}")
        m.bar(f"ve{s}")
    for name in ("s", "o"):
        m.bar(name)
    for name in ("sf", "p"):
        m.bar(name, ROWS)
    roles = {"producer": producer(m, items), "mma": mma_issuer(m)}
    roles.update({f"rows{w}": query_rows(m, w) for w in range(ROWS)})
    simulate(m, roles, random.Random(seed))


def random_items(rng, max_blocks=5):
    return [(rng.random() < 0.35, rng.randint(1, max_blocks)) for _ in range(rng.randint(1, 7))]


@pytest.mark.parametrize("seed", range(40))
def test_random_item_sequences_and_schedules(seed):
    rng = random.Random(2000 + seed)
    items = random_items(rng)
    for sched in range(15):
        run(items, seed * 100 + sched)


def test_edge_sequences():
    """One-block items (the diagonal block only), kinds alternating, long runs."""
    cases = [
        [(False, 1)] * 6,
        [(True, 1)] * 6,
        [(False, 1), (True, 1)] * 4,
        [(True, 3), (False, 1), (True, 2), (False, 4), (False, 1)],
        [(False, 5)] * 3,
        [(True, 5), (True, 4), (False, 2), (True, 1)],
    ]
    for i, items in enumerate(cases):
        for sched in range(40):
            run(items, 9000 + 100 * i + sched)


def _caught(seed):
    import tests.test_fwd_schedule_model as mod
    rng = random.Random(seed)
    for trial in range(300):
        try:
            mod.run(random_items(rng, 4), trial)
        except ModelError:
            return True
    return False


@pytest.mark.parametrize("fn_name,old,new", [
    # S_{j+1} issued before the rows copied S_j out of TMEM
    ("mma_issuer", 'yield W("sf", go + j, (go + j) & 1)', 'pass'),
    # P_j written before P.V_{j-1} has read P_{j-1}
    ("query_rows", 'yield W("o", go + j - 1, (go + j - 1) & 1)', 'pass'),
    # a replaced head's W buffer rewritten before its P.V ran
    ("query_rows", "if g >= 2:\n", "if False:\n"),
    # a K stage reloaded before its S MMA ran
    ("producer", 'yield W(f"ke{s}", u - 1, (u & 1) ^ 1)', 'yield from ()'),
    # the next-but-one item's Q loaded over a Q still in use
    ("producer", 'yield W(f"qe{b}", (nq >> 1) - 1, ((nq >> 1) & 1) ^ 1)', 'pass'),
    # a replaced block's W inputs staged over those the rows still build from
    ("producer", "if gw >= 2:\n", "if False:\n"),
    # the rows build W before its inputs have landed
    ("query_rows", 'yield W(f"wf{g & 1}", g >> 1, (g >> 1) & 1)', 'pass'),
    # an O box staged over the previous one before its store has read it
    ("query_rows", "if ns > 0:\n", "if False:\n"),
], ids=["no_sf", "no_o", "no_ob", "no_ke", "no_qe", "no_pb_stage", "no_wf", "no_store_read"])
def test_model_catches_planted_mistakes(monkeypatch, fn_name, old, new):
    """Each planted mistake in the protocol is caught on some schedule."""
    import tests.test_fwd_schedule_model as mod
    mutate(monkeypatch, mod, fn_name, old, new)
    assert _caught(3)
