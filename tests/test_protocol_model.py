"""A model of the tensor-core attention kernels' synchronisation, checked on the CPU.

This models the barrier protocols of k_bwd_dq_persist, k_bwd_dkdv_persist and
k_attn_fwd_sm100 as their source comments state them; it does not run the kernels. Each role is a
Python generator: the TMA producer, every MMA-issuing warp, and the elementwise
warps taken as one agent. A random scheduler interleaves the roles, the
asynchronous TMA copies and the MMAs. MMAs complete in issue order per issuing
warp, and a commit arrives once every earlier MMA of its warp is complete.

Under thousands of random schedules, the test checks:
- no schedule deadlocks;
- every parity wait finds its barrier either at the awaited phase or one phase
  past it (a barrier two phases ahead, or one behind, would fool a parity test);
- no MMA, elementwise step, copy or epilogue meets a TMEM buffer, ring stage or
  accumulator that holds another granule's data.
"""
import random

import pytest


class Bar:
    """An mbarrier: `count` arrivals complete a phase; `done` phases completed.
    `name` is the barrier's name in the kernel (a family shares one)."""

    def __init__(self, count=1, name=""):
        self.count, self.left, self.done, self.name = count, count, 0, name

    def arrive(self):
        self.left -= 1
        assert self.left >= 0
        if self.left == 0:
            self.done += 1
            self.left = self.count


class Deadlock(AssertionError):
    pass


class Sim:
    """Random interleaving of agents (generators) and asynchronous work."""

    def __init__(self, seed, drop=None):
        self.rng = random.Random(seed)
        self.agents = {}            # name -> [generator, pending action]
        self.fifo = {}              # issuing warp -> queued MMA / commit entries
        self.copies = []            # in-flight TMA copies: (fn, barrier)
        self.drop = drop            # (agent, barrier name): those waits pass at once
        self.sites = set()          # (agent, barrier name) of every wait met

    def add(self, name, gen):
        self.agents[name] = [gen, None]
        self.fifo.setdefault(name, [])

    # actions a role yields
    @staticmethod
    def wait(bar, phase):
        return ("wait", bar, phase)

    def _advance(self, name):
        gen, _ = self.agents[name]
        try:
            self.agents[name][1] = next(gen)
        except StopIteration:
            self.agents[name][1] = "end"

    def _enabled(self, name):
        act = self.agents[name][1]
        if act == "end":
            return False
        if act[0] == "until":                      # a plain condition (e.g. a warp reconverging)
            return act[1]()
        if act[0] == "wait":
            _, bar, n = act
            self.sites.add((name, bar.name))
            if (name, bar.name) == self.drop:
                return True
            # a parity wait for phase n is only sound while the barrier has
            # completed n or n + 1 phases
            assert n <= bar.done <= n + 1, (name, n, bar.done)
            return bar.done >= n + 1
        return True

    def run(self, max_steps=200000):
        for name in self.agents:
            self._advance(name)
        for _ in range(max_steps):
            choices = [("agent", n) for n in self.agents if self._enabled(n)]
            choices += [("mma", w) for w, q in self.fifo.items() if q]
            choices += [("copy", i) for i in range(len(self.copies))]
            if not choices:
                if all(a[1] == "end" for a in self.agents.values()):
                    return
                raise Deadlock({n: a[1] for n, a in self.agents.items() if a[1] != "end"})
            kind, key = self.rng.choice(choices)
            if kind == "agent":
                act = self.agents[key][1]
                if act[0] == "until":
                    pass
                elif act[0] == "do":
                    act[1]()
                elif act[0] == "mma":               # issue: queue behind this warp's earlier work
                    self.fifo[key].append(("mma", act[1]))
                elif act[0] == "commit":
                    self.fifo[key].append(("commit", act[1]))
                elif act[0] == "copy":
                    self.copies.append((act[1], act[2]))
                self._advance(key)
            elif kind == "mma":
                what, arg = self.fifo[key].pop(0)
                if what == "mma":
                    arg()                           # the MMA runs: its checks and writes
                else:
                    arg.arrive()                    # every earlier MMA of the warp is done
            else:
                fn, bar = self.copies.pop(key)
                fn()
                bar.arrive()
        raise AssertionError("schedule did not finish")


def make_items(rng, n_items):
    """Granule counts of one CTA's items, empty ones included."""
    return [rng.choice([0, 1, 1, 2, 3, 5, 8]) for _ in range(n_items)]


# ---------------------------------------------------------------------------- dK/dV
def dkdv_model(seed, items, nst, drop=None):
    """k_bwd_dkdv_persist: producer (ring lanes and stationary-tile lanes of one
    warp, reconverging once an item), warp 1 S^T/dP^T, warp 2 dV/dK, and the
    elementwise warpgroups with the epilogue."""
    sim = Sim(seed, drop)
    W = Sim.wait
    full0 = [Bar(name="full0") for _ in range(nst)]
    fullx = [Bar(name="fullx") for _ in range(nst)]
    empty = [Bar(name="empty") for _ in range(nst)]
    prod, elem = [Bar(name="prod") for _ in range(2)], [Bar(name="elem") for _ in range(2)]
    kv_done = [Bar(name="kv_done") for _ in range(2)]
    rows_full, rows_empty = [Bar(name="rows_full") for _ in range(2)], [Bar(name="rows_empty") for _ in range(2)]
    stat, kv_free, fin = Bar(name="stat"), Bar(name="kv_free"), Bar(name="fin")
    st = dict(ring=[None] * nst, xs=[None] * nst, tmem=[None, None], kvtile=None, acc="free",
              rows=[None, None], sdp_done=set(), dvdk_done=set(), item_sync={})
    # granule numbering over the CTA's items, and each item's first granule
    first, G = [], 0
    for ng in items:
        first.append(G)
        G += ng
    nonempty = [j for j, ng in enumerate(items) if ng > 0]
    kq_of = {j: k for k, j in enumerate(nonempty)}

    def sync(j, who):
        st["item_sync"].setdefault(j, set()).add(who)
        return ("until", lambda: len(st["item_sync"][j]) == 2)

    def ring_lanes():
        for j, ng in enumerate(items):
            if j >= 2:
                yield W(rows_empty[j & 1], (j >> 1) - 1)

            def write_rows(j=j):
                st["rows"][j & 1] = j
                rows_full[j & 1].arrive()
            yield ("do", write_rows)
            for g in range(ng):
                Gg = first[j] + g
                s, cyc = Gg % nst, Gg // nst
                if cyc >= 1:
                    yield W(empty[s], cyc - 1)

                def land(Gg=Gg, s=s):
                    assert Gg < nst or (Gg - nst) in st["dvdk_done"], ("ring stage reused early", Gg)
                    st["ring"][s] = Gg

                def land_x(Gg=Gg, s=s):
                    assert Gg < nst or (Gg - nst) in st["dvdk_done"]
                    st["xs"][s] = Gg
                yield ("copy", land, full0[s])
                yield ("copy", land_x, fullx[s])
            yield sync(j, "ring")

    def stat_lanes():
        for j, ng in enumerate(items):
            if ng > 0:
                kq = kq_of[j]
                if kq >= 1:
                    yield W(kv_free, kq - 1)

                def land(kq=kq):
                    prev = nonempty[kq - 1] if kq >= 1 else None
                    if prev is not None:      # every S^T/dP^T MMA of the previous item complete
                        assert all(first[prev] + g in st["sdp_done"] for g in range(items[prev]))
                    st["kvtile"] = kq
                yield ("copy", land, stat)
            yield sync(j, "stat")

    def warp1():
        for j in nonempty:
            kq, ng = kq_of[j], items[j]
            yield W(stat, kq)
            for g in range(ng):
                Gg = first[j] + g
                s, b, u = Gg % nst, Gg & 1, Gg >> 1
                yield W(full0[s], Gg // nst)
                if Gg >= 2:
                    yield W(kv_done[b], u - 1)

                def mma(Gg=Gg, s=s, b=b, kq=kq):
                    assert st["ring"][s] == Gg and st["kvtile"] == kq
                    assert st["tmem"][b] in (None, ("done", Gg - 2)), ("S^T over unread P^T", Gg, st["tmem"][b])
                    st["tmem"][b] = ("S", Gg)
                    st["sdp_done"].add(Gg)
                yield ("mma", mma)
                yield ("commit", prod[b])
                if g == ng - 1:
                    yield ("commit", kv_free)

    def warp2():
        for j in nonempty:
            ng = items[j]
            for g in range(ng):
                Gg = first[j] + g
                s, b, u = Gg % nst, Gg & 1, Gg >> 1
                yield W(elem[b], u)

                def mma(Gg=Gg, s=s, b=b, j=j, g=g):
                    assert st["tmem"][b] == ("P", Gg) and st["ring"][s] == Gg
                    if g == 0:
                        assert st["acc"] == "free", ("dK/dV overwritten before the epilogue", j)
                        st["acc"] = (j, 1)
                    else:
                        assert st["acc"] == (j, g)
                        st["acc"] = (j, g + 1)
                    st["tmem"][b] = ("done", Gg)
                    st["dvdk_done"].add(Gg)
                yield ("mma", mma)
                yield ("commit", empty[s])
                yield ("commit", kv_done[b])
            yield ("commit", fin)

    def elementwise():
        kf = 0
        for j, ng in enumerate(items):
            yield W(rows_full[j & 1], j >> 1)

            def read_rows(j=j):
                assert st["rows"][j & 1] == j, ("selection rows", j)
            yield ("do", read_rows)
            for g in range(ng):
                Gg = first[j] + g
                s, b, u = Gg % nst, Gg & 1, Gg >> 1
                yield W(prod[b], u)
                yield W(fullx[s], Gg // nst)

                def step(Gg=Gg, s=s, b=b):
                    assert st["tmem"][b] == ("S", Gg) and st["xs"][s] == Gg
                    st["tmem"][b] = ("P", Gg)
                yield ("do", step)
                yield ("do", lambda b=b: elem[b].arrive())
            yield ("do", lambda j=j: rows_empty[j & 1].arrive())
            if ng > 0:
                yield W(fin, kf)
                kf += 1

                def epilogue(j=j, ng=ng):
                    assert st["acc"] == (j, ng), ("epilogue", j, st["acc"])
                    st["acc"] = "free"
                yield ("do", epilogue)

    for name, gen in (("ring", ring_lanes()), ("stat", stat_lanes()), ("w1", warp1()), ("w2", warp2()),
                      ("elem", elementwise())):
        sim.add(name, gen)
    sim.run()
    assert len(st["dvdk_done"]) == sum(items)
    return sim


@pytest.mark.parametrize("nst", [2, 3, 4, 5])
def test_dkdv_protocol_random_schedules(nst):
    rng = random.Random(nst)
    for trial in range(150):
        items = make_items(rng, rng.randint(1, 7))
        dkdv_model(1000 * nst + trial, items, nst)


# ---------------------------------------------------------------------------- dQ
def dq_model(seed, items, nst, drop=None):
    """k_bwd_dq_persist: producer (selection rows, K and V ring), warp 1 S, warp 10
    dP, warp 11 dQ, and the elementwise warpgroups, which write the next non-empty
    item's Q and dO into TMEM and run the epilogue."""
    sim = Sim(seed, drop)
    W = Sim.wait
    full0 = [Bar(name="full0") for _ in range(nst)]
    empty = [Bar(name="empty") for _ in range(nst)]
    prod = [Bar(2, "prod") for _ in range(2)]   # the S and the dP issuer each commit
    elem, dq_done = [Bar(name="elem") for _ in range(2)], [Bar(name="dq_done") for _ in range(2)]
    rows_full, rows_empty = [Bar(name="rows_full") for _ in range(2)], [Bar(name="rows_empty") for _ in range(2)]
    qdo_full, fin = Bar(name="qdo_full"), Bar(name="fin")
    st = dict(ring=[None] * nst, S=[None, None], P=[None, None], qdo=None, acc="free", rows=[None, None],
              s_done=set(), p_done=set(), q_done=set())
    first, G = [], 0
    for ng in items:
        first.append(G)
        G += ng
    nonempty = [j for j, ng in enumerate(items) if ng > 0]
    kq_of = {j: k for k, j in enumerate(nonempty)}

    def producer():
        for j, ng in enumerate(items):
            if j >= 2:
                yield W(rows_empty[j & 1], (j >> 1) - 1)

            def write_rows(j=j):
                st["rows"][j & 1] = j
                rows_full[j & 1].arrive()
            yield ("do", write_rows)
            for g in range(ng):
                Gg = first[j] + g
                s, cyc = Gg % nst, Gg // nst
                if cyc >= 1:
                    yield W(empty[s], cyc - 1)

                def land(Gg=Gg, s=s):
                    old = Gg - nst           # the stage's previous granule: S, dP and dQ all read it
                    assert old < 0 or {old} <= st["s_done"] & st["p_done"] & st["q_done"], ("ring", Gg)
                    st["ring"][s] = Gg
                yield ("copy", land, full0[s])

    def s_or_dp(which):
        buf, done = ("S", "s_done") if which == "S" else ("P", "p_done")
        for j in nonempty:
            kq, ng = kq_of[j], items[j]
            yield W(qdo_full, kq)
            for g in range(ng):
                Gg = first[j] + g
                s, b, u = Gg % nst, Gg & 1, Gg >> 1
                yield W(full0[s], Gg // nst)
                if Gg >= 2:
                    yield W(elem[b], u - 1)
                    if which == "S":             # dS lives over the S columns
                        yield W(dq_done[b], u - 1)

                def mma(Gg=Gg, s=s, b=b, kq=kq):
                    assert st["ring"][s] == Gg and st["qdo"] == kq, (which, Gg)
                    free = (None, ("dS read", Gg - 2)) if which == "S" else (None, ("read", Gg - 2))
                    assert st[buf][b] in free, (which, "over unconsumed columns", Gg, st[buf][b])
                    st[buf][b] = (which, Gg)
                    st[done].add(Gg)
                yield ("mma", mma)
                yield ("commit", prod[b])

    def warp11():
        for j in nonempty:
            ng = items[j]
            for g in range(ng):
                Gg = first[j] + g
                s, b, u = Gg % nst, Gg & 1, Gg >> 1
                yield W(elem[b], u)

                def mma(Gg=Gg, s=s, b=b, j=j, g=g):
                    assert st["S"][b] == ("dS", Gg) and st["ring"][s] == Gg
                    if g == 0:
                        assert st["acc"] == "free", ("dQ overwritten before the epilogue", j)
                        st["acc"] = (j, 1)
                    else:
                        assert st["acc"] == (j, g)
                        st["acc"] = (j, g + 1)
                    st["S"][b] = ("dS read", Gg)
                    st["q_done"].add(Gg)
                yield ("mma", mma)
                yield ("commit", empty[s])
                yield ("commit", dq_done[b])
            yield ("commit", fin)

    def elementwise():
        kf = 0
        loaded = [0]

        def q_ahead(itn):
            # Q and dO of a non-empty item: every S/dP MMA of the items before it complete
            if itn < len(items) and items[itn] > 0:
                def write(itn=itn):
                    kq = kq_of[itn]
                    for prev in nonempty[:kq]:
                        for g in range(items[prev]):
                            assert first[prev] + g in st["s_done"] and first[prev] + g in st["p_done"], "Q/dO"
                    st["qdo"] = kq
                    qdo_full.arrive()
                    loaded[0] += 1
                yield ("do", write)
        yield from q_ahead(0)
        for j, ng in enumerate(items):
            yield W(rows_full[j & 1], j >> 1)

            def read_rows(j=j):
                assert st["rows"][j & 1] == j, ("selection rows", j)
            yield ("do", read_rows)
            for g in range(ng):
                Gg = first[j] + g
                b, u = Gg & 1, Gg >> 1
                yield W(prod[b], u)

                def step(Gg=Gg, b=b):
                    assert st["S"][b] == ("S", Gg) and st["P"][b] == ("P", Gg)
                    st["S"][b] = ("dS", Gg)
                    st["P"][b] = ("read", Gg)
                    elem[b].arrive()
                yield ("do", step)
            yield ("do", lambda j=j: rows_empty[j & 1].arrive())
            yield from q_ahead(j + 1)
            if ng > 0:
                yield W(fin, kf)
                kf += 1

                def epilogue(j=j, ng=ng):
                    assert st["acc"] == (j, ng), ("epilogue", j, st["acc"])
                    st["acc"] = "free"
                yield ("do", epilogue)

    for name, gen in (("producer", producer()), ("w1", s_or_dp("S")), ("w10", s_or_dp("P")), ("w11", warp11()),
                      ("elem", elementwise())):
        sim.add(name, gen)
    sim.run()
    assert len(st["q_done"]) == sum(items)
    return sim


@pytest.mark.parametrize("nst", [2, 3, 4, 5])
def test_dq_protocol_random_schedules(nst):
    rng = random.Random(100 + nst)
    for trial in range(150):
        items = make_items(rng, rng.randint(1, 7))
        dq_model(2000 * nst + trial, items, nst)


# ---------------------------------------------------------------------------- dQ from stored dS
def dq_ds_model(seed, items, nst, drop=None):
    """k_bwd_dq_ds: the copy lanes (K and both dS^T blocks of a granule into one
    ring stage), the MMA warp (dQ += dS K into accumulator b = k & 1 of non-empty
    item k) and the epilogue warps, which read accumulator b and free it."""
    sim = Sim(seed, drop)
    W = Sim.wait
    full = [Bar(name="full") for _ in range(nst)]
    empty = [Bar(name="empty") for _ in range(nst)]
    fin = [Bar(name="fin") for _ in range(2)]
    acc_free = [Bar(name="acc_free") for _ in range(2)]
    st = dict(ring=[None] * nst, acc=["free", "free"], done=set(), stored=[])
    first, G = [], 0
    for ng in items:
        first.append(G)
        G += ng
    nonempty = [j for j, ng in enumerate(items) if ng > 0]
    kq_of = {j: k for k, j in enumerate(nonempty)}

    def producer():
        for j, ng in enumerate(items):
            for g in range(ng):
                Gg = first[j] + g
                s, cyc = Gg % nst, Gg // nst
                if cyc >= 1:
                    yield W(empty[s], cyc - 1)

                def land(Gg=Gg, s=s):
                    assert Gg < nst or (Gg - nst) in st["done"], ("ring stage reused early", Gg)
                    st["ring"][s] = Gg
                yield ("copy", land, full[s])

    def mma_warp():
        for j in nonempty:
            kq, ng = kq_of[j], items[j]
            b = kq & 1
            if kq >= 2:
                yield W(acc_free[b], (kq >> 1) - 1)
            for g in range(ng):
                Gg = first[j] + g
                s = Gg % nst
                yield W(full[s], Gg // nst)

                def mma(Gg=Gg, s=s, b=b, j=j, g=g):
                    assert st["ring"][s] == Gg, ("MMA before its operands", Gg)
                    if g == 0:
                        assert st["acc"][b] == "free", ("dQ over an unread accumulator", j)
                        st["acc"][b] = (j, 1)
                    else:
                        assert st["acc"][b] == (j, g)
                        st["acc"][b] = (j, g + 1)
                    st["done"].add(Gg)
                yield ("mma", mma)
                yield ("commit", empty[s])
            yield ("commit", fin[b])

    def epilogue():
        for j, ng in enumerate(items):
            if ng == 0:
                yield ("do", lambda j=j: st["stored"].append(j))      # zeros, no TMEM
                continue
            kq = kq_of[j]
            b = kq & 1
            yield W(fin[b], kq >> 1)

            def store(j=j, ng=ng, b=b):
                assert st["acc"][b] == (j, ng), ("epilogue", j, st["acc"][b])
                st["acc"][b] = "free"
                st["stored"].append(j)
                acc_free[b].arrive()
            yield ("do", store)

    for name, gen in (("producer", producer()), ("mma", mma_warp()), ("epi", epilogue())):
        sim.add(name, gen)
    sim.run()
    assert st["stored"] == list(range(len(items))) and len(st["done"]) == sum(items)
    return sim


@pytest.mark.parametrize("nst", [2, 3, 6, 8])
def test_dq_ds_protocol_random_schedules(nst):
    rng = random.Random(300 + nst)
    for trial in range(200):
        items = make_items(rng, rng.randint(1, 9))
        dq_ds_model(3000 * nst + trial, items, nst)


# ---------------------------------------------------------------------------- forward
def fwd_model(seed, nch, p_quarter=lambda g: 2 * g, drop=None):
    """k_attn_fwd_sm100, one CTA (one item): producer (Q once; K and V of each chunk
    in one buffer each), warp 1 (S = Q K^T into the one S buffer, then O += P V),
    and the two softmax warpgroups as two agents. The S buffer is tracked in four
    32-column quarters; warpgroup g reads quarters 2g and 2g+1 (its key granule)
    twice, with the row-maximum exchange between the reads, and writes its P into
    quarter p_quarter(g)."""
    sim = Sim(seed, drop)
    W = Sim.wait
    bar_q, bar_kf, bar_ke = Bar(name="bar_q"), Bar(name="bar_kf"), Bar(name="bar_ke")
    bar_vf, bar_ve = Bar(name="bar_vf"), Bar(name="bar_ve")
    bar_s, bar_p, bar_o = Bar(name="bar_s"), Bar(2, "bar_p"), Bar(name="bar_o")
    st = dict(K=None, V=None, S=[None] * 4, O=[], xmax=[[None, None], [None, None]], xbar={}, pv_done=set())

    def producer_k():
        for c in range(nch):
            if c > 0:
                yield W(bar_ke, c - 1)

            def land(c=c):
                assert c == 0 or c - 1 in st["s_done"], "K overwritten before S read it"
                st["K"] = c
            yield ("copy", land, bar_kf)

    def producer_v():
        for c in range(nch):
            if c > 0:
                yield W(bar_ve, c - 1)

            def land(c=c):
                assert c == 0 or c - 1 in st["pv_done"], "V overwritten before PV read it"
                st["V"] = c
            yield ("copy", land, bar_vf)

    st["s_done"] = set()

    def mma_warp():
        yield ("copy", lambda: st.update(Q=True), bar_q)
        yield W(bar_q, 0)
        for c in range(nch):
            yield W(bar_kf, c)

            def s_mma(c=c):
                assert st.get("Q") and st["K"] == c
                # the previous chunk's P has been read by PV(c - 1), issued earlier by this warp
                assert all(q is None or q[0] == "read" for q in st["S"]), ("S over unread P", c, st["S"])
                st["S"] = [("S", c)] * 4
                st["s_done"].add(c)
            yield ("mma", s_mma)
            yield ("commit", bar_ke)
            yield ("commit", bar_s)
            yield W(bar_p, c)
            yield W(bar_vf, c)

            def pv_mma(c=c):
                assert st["V"] == c
                for g in range(2):
                    assert st["S"][p_quarter(g)] == ("P", c, g), ("PV reads", c, g, st["S"])
                st["S"] = [("read", c)] * 4
                st["O"].append(c)
                st["pv_done"].add(c)
            yield ("mma", pv_mma)
            yield ("commit", bar_ve)
        yield ("commit", bar_o)

    def softmax(g):
        for c in range(nch):
            yield W(bar_s, c)

            def pass1(c=c):
                for q in (2 * g, 2 * g + 1):
                    assert st["S"][q] == ("S", c), ("pass 1 reads", g, c, st["S"])
                if c > 0:                        # a rescale of O needs PV(c - 1) complete
                    assert c - 1 in st["pv_done"]
                st["xmax"][c & 1][g] = c
                st["xbar"].setdefault(c, set()).add(g)
            yield ("do", pass1)
            yield ("until", lambda c=c: len(st["xbar"][c]) == 2)     # named barrier of both warpgroups

            def pass2(c=c):
                assert st["xmax"][c & 1][g ^ 1] == c, ("row maximum exchange", g, c)
                for q in (2 * g, 2 * g + 1):
                    assert st["S"][q] in (("S", c), ("P", c, g)), ("pass 2 reads", g, c, st["S"])
                st["S"][p_quarter(g)] = ("P", c, g)
                bar_p.arrive()
            yield ("do", pass2)
        yield W(bar_o, 0)

        def epilogue():
            assert st["O"] == list(range(nch))
        yield ("do", epilogue)

    for name, gen in (("k", producer_k()), ("v", producer_v()), ("mma", mma_warp()), ("wg0", softmax(0)),
                      ("wg1", softmax(1))):
        sim.add(name, gen)
    sim.run()
    return sim


def test_fwd_protocol_random_schedules():
    for trial in range(400):
        fwd_model(trial, 1 + trial % 9)


def test_fwd_model_catches_p_over_the_other_granules_columns():
    """P of warpgroup 1 written over S columns 32-63, which warpgroup 0 reads again in
    its second pass: the layout a GPU parity run once rejected."""
    with pytest.raises(AssertionError):
        for trial in range(400):
            fwd_model(trial, 1 + trial % 9, p_quarter=lambda g: g)


# ---------------------------------------------------------------------------- every wait is needed
def _catches(run):
    """True when some random schedule breaks a check (a hazard, an unsound parity
    wait or a deadlock)."""
    try:
        run()
    except AssertionError:
        return True
    return False


def _items_runs(model, base, nst):
    rng = random.Random(base)
    cases = [(base + t, make_items(rng, rng.randint(2, 9))) for t in range(300)]
    return lambda drop: [model(seed, items, nst, drop) for seed, items in cases]


MODELS = {
    "dkdv": lambda: _items_runs(dkdv_model, 7000, 3),
    "dq": lambda: _items_runs(dq_model, 8000, 3),
    "dq_ds": lambda: _items_runs(dq_ds_model, 9000, 3),
    "fwd": lambda: (lambda drop: [fwd_model(t, 1 + t % 9, drop=drop) for t in range(400)]),
}


# Waits that another wait of the same role already implies.  In k_bwd_dq_persist
# the S issuer waits elem(b) and then dq_done(b) of the buffer's previous use;
# the dQ MMA that dq_done(b) tracks was itself issued only after that elem(b)
# phase, so the first wait adds nothing to the second.
REDUNDANT = {"dq": [("w1", "elem")]}


@pytest.mark.parametrize("model", list(MODELS))
def test_dropping_any_wait_is_caught(model):
    """Each (role, barrier) wait of the model, dropped on its own, lets some
    schedule break a check, except the waits listed as implied by another: the
    model's checks see what each wait guards."""
    runs = MODELS[model]()
    sites = set()
    for sim in runs(None):
        sites |= sim.sites
    assert sites
    missed = [site for site in sorted(sites) if not _catches(lambda site=site: runs(site))]
    assert missed == REDUNDANT.get(model, []), missed
