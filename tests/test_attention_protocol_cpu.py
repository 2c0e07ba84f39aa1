"""Randomized models of the mbarrier protocols of the two tcgen05 attention
kernels (csrc/attention_tc.cu, csrc/attention_tc_long.cu), run on the CPU.

Each role of a kernel (TMA producer, MMA issuer, softmax warps, output warps) is
a coroutine that performs the kernel's waits, arrivals and commits in the
kernel's order; asynchronous completions (TMA bytes, tcgen05.commit) are
delivered later in random order per barrier, and roles run at random relative
speeds.  An mbarrier is modelled as the hardware defines it: a phase completes
after `count` arrivals and a parity wait returns as soon as the current phase's
parity differs from the one asked for -- so a role that falls two phases behind
would see a false completion.  The checks:
  * every wait that returns observes the phase of the item it expects (phases
    carry the item that completed them);
  * a phase never mixes arrivals of two items;
  * tensor memory: no product overwrites columns another role still reads
    (scores of an item stay until its softmax is done, O until the output warps
    have read it, and O of the long kernel only after block 0's scores are read);
  * every run finishes (no deadlock).
A planted protocol mistake (checked below) makes these checks fail, so they are
not vacuous.
"""
import random

import pytest


class Bar:
    def __init__(self, name, count):
        self.name, self.count, self.arrived, self.phase, self.tags, self.cur = name, count, 0, 0, [], []

    def arrive(self, tag):
        self.cur.append(tag)
        self.arrived += 1
        if self.arrived == self.count:
            assert len(set(self.cur)) == 1, (self.name, "phase mixes items", self.cur)
            self.tags.append(self.cur[0])
            self.cur, self.arrived = [], 0
            self.phase += 1

    def test(self, parity):
        return (self.phase & 1) != parity


class Sim:
    def __init__(self, seed):
        self.rnd = random.Random(seed)
        self.bars, self.pending = {}, []

    def bar(self, name, count):
        self.bars[name] = Bar(name, count)

    def commit(self, name, tag):
        self.pending.append((name, tag))

    def wait(self, name, parity, tag=None):
        b = self.bars[name]
        while not b.test(parity):
            yield
        if tag is not None:
            idx = b.phase - 1 if ((b.phase - 1) & 1) == parity else b.phase - 2
            assert idx >= 0 and b.tags[idx] == tag, (name, "wait saw", b.tags[idx] if idx >= 0 else None, "want", tag)

    def run(self, roles):
        speed = {id(r): self.rnd.choice([1.0, 1.0, 0.1, 0.02]) for r in roles}
        alive, steps = list(roles), 0
        while alive or self.pending:
            steps += 1
            assert steps < 2_000_000, "deadlock"
            if self.pending and (not alive or self.rnd.random() < 0.3):
                name = self.pending[self.rnd.randrange(len(self.pending))][0]
                k = min(i for i, p in enumerate(self.pending) if p[0] == name)  # in order per barrier
                n, t = self.pending.pop(k)
                self.bars[n].arrive(t)
                continue
            if not alive:
                continue
            r = self.rnd.choice(alive)
            if self.rnd.random() > speed[id(r)]:
                continue
            try:
                next(r)
            except StopIteration:
                alive.remove(r)


# ----------------------------------------------------------------- short kernel --
# One item per (sequence, head), four TMEM buffers, Q/K and V stages with the
# buffer's index; a stage is released by the S (Q/K) or O (V) completion of the
# item four back.  The producer loads Q/K of every item and V of items 0..3; one
# output warp loads V of item i + 4 once it has seen O of item i complete.  Two
# softmax groups take alternate items.  Two issuing threads: one issues the S
# products in item order, the other the O products.
# planted: True loads V of item i + 4 before O of item i is complete; "s_early"
# issues S into a buffer without waiting for the output warps to have read its
# previous O.
def short_kernel(n_items, seed, planted=False):
    NB = 4
    sim = Sim(seed)
    for i in range(NB):
        for n, c in (("qk_full", 1), ("v_full", 1), ("s_full", 1), ("p_full", 4), ("o_full", 1), ("o_empty", 4)):
            sim.bar(f"{n}{i}", c)
    tmem = {}  # buffer -> item whose S/P/O it holds

    def load_v(n):
        if n >= NB:
            assert sim.bars[f"o_full{n % NB}"].phase > (n - NB) // NB, "V stage reused before O read it"
        sim.commit(f"v_full{n % NB}", ("v", n))

    def producer():
        for nq in range(n_items):
            yield from sim.wait(f"s_full{nq % NB}", ((nq // NB) & 1) ^ 1)
            if nq >= NB:
                assert sim.bars[f"s_full{nq % NB}"].phase > (nq - NB) // NB, "Q/K stage reused before S read it"
            sim.commit(f"qk_full{nq % NB}", ("qk", nq))
            if nq < NB:
                load_v(nq)
            yield

    def mma_s():
        for ns in range(n_items):
            tb = ns % NB
            yield from sim.wait(f"qk_full{tb}", (ns // NB) & 1, ("qk", ns))
            if planted != "s_early":
                yield from sim.wait(f"o_empty{tb}", ((ns // NB) & 1) ^ 1)
            assert tmem.get(tb) in (None, ("read", ns - NB)), ("S over a buffer still in use", tmem.get(tb))
            tmem[tb] = ("s", ns)
            sim.commit(f"s_full{tb}", ("s", ns))
            yield

    def mma_o():
        for no in range(n_items):
            tb = no % NB
            yield from sim.wait(f"p_full{tb}", (no // NB) & 1, ("p", no))
            yield from sim.wait(f"v_full{tb}", (no // NB) & 1, ("v", no))
            assert tmem.get(tb) == ("s", no), ("O product into a buffer holding", tmem.get(tb), "for item", no)
            sim.commit(f"o_full{tb}", ("o", no))
            yield

    def softmax(g):
        for i in range(g, n_items, 2):
            tb = i % NB
            yield from sim.wait(f"s_full{tb}", (i // NB) & 1, ("s", i))
            assert tmem[tb] == ("s", i)
            yield
            sim.bars[f"p_full{tb}"].arrive(("p", i))

    def output(q):
        for i in range(n_items):
            tb = i % NB
            if planted is True and q == 2 and i + NB < n_items:
                load_v(i + NB)  # the planted mistake: before O of item i is complete
            yield from sim.wait(f"o_full{tb}", (i // NB) & 1, ("o", i))
            if planted is not True and q == 2 and i + NB < n_items:
                load_v(i + NB)
            yield from sim.wait(f"p_full{tb}", (i // NB) & 1, ("p", i))
            yield
            sim.bars[f"o_empty{tb}"].arrive(("e", i))
            if sim.bars[f"o_empty{tb}"].arrived == 0:
                tmem[tb] = ("read", i)

    sim.run([producer(), mma_s(), mma_o()] + [softmax(g) for g in range(2) for _ in range(4)] +
            [output(q) for q in range(4)])


# ------------------------------------------------------------------ long kernel --
# One item per (sequence, 128-query block, head); all of its scores in TMEM
# (key block j in columns 128j..), O in columns 64..127.  Softmax half w owns
# key blocks w, w+2 and exchanges row maxima with the other half when both own a
# block.  S of an item waits until the output warps have read the previous O.
def long_kernel(items, seed, planted=False):
    NVS = 2
    sim = Sim(seed)
    for n, c in (("qk_full", 1), ("qk_empty", 1), ("o_full", 1), ("o_empty", 4)):
        sim.bar(n, c)
    for s in range(NVS):
        sim.bar(f"v_full{s}", 1)
        sim.bar(f"v_empty{s}", 1)
    for j in range(4):
        sim.bar(f"s_full{j}", 1)
        sim.bar(f"p_full{j}", 4)
    for q in range(4):
        sim.bar(f"x{q}", 2)
    st = {"item": None, "o_read": -1, "s0_read": 0, "p": {}, "xmax": set(), "xsum": set()}

    def producer():
        for i, (nkb, _) in enumerate(items):
            yield from sim.wait("qk_empty", (i & 1) ^ 1)
            sim.commit("qk_full", ("qk", i))
            yield from sim.wait(f"v_empty{i % NVS}", ((i // NVS) & 1) ^ 1)
            sim.commit(f"v_full{i % NVS}", ("v", i))

    def mma():
        par = 0
        for i, (nkb, _) in enumerate(items):
            yield from sim.wait("qk_full", i & 1, ("qk", i))
            if not planted:
                yield from sim.wait("o_empty", (i & 1) ^ 1, ("e", i - 1) if i else None)
                assert st["o_read"] == i - 1
            st["item"] = i
            for j in range(nkb):
                sim.commit(f"s_full{j}", ("s", i))
            sim.commit("qk_empty", ("qk-free", i))
            yield from sim.wait(f"v_full{i % NVS}", (i // NVS) & 1, ("v", i))
            for j in range(nkb):  # O products in block order: block 0 first
                yield from sim.wait(f"p_full{j}", (par >> j) & 1, ("p", i))
                assert st["p"].get((i, j)) == 4
                if j == 0:
                    assert st["s0_read"] == 4 * (i + 1), "O written over block 0's unread scores"
            sim.commit("o_full", ("o", i))
            sim.commit(f"v_empty{i % NVS}", ("v-free", i))
            par ^= (1 << nkb) - 1

    def softmax(half, quad):
        par = xpar = 0
        for i, (nkb, live_q) in enumerate(items):
            live = live_q[quad]
            for j in range(half, nkb, 2):
                yield from sim.wait(f"s_full{j}", (par >> j) & 1, ("s", i))
                assert st["item"] == i
            if live and nkb >= 2:
                st["xmax"].add((i, half, quad))
                sim.bars[f"x{quad}"].arrive(("x", i))
                yield from sim.wait(f"x{quad}", xpar, ("x", i))
                xpar ^= 1
                assert (i, half ^ 1, quad) in st["xmax"]
            for j in range(half, nkb, 2):
                assert st["item"] == i, "scores overwritten during the softmax"
                yield
                if j == 0:
                    st["s0_read"] += 1
                if j + 2 >= nkb and live:
                    st["xsum"].add((i, half, quad))
                st["p"][(i, j)] = st["p"].get((i, j), 0) + 1
                sim.bars[f"p_full{j}"].arrive(("p", i))
            par ^= (1 << nkb) - 1

    def output(quad):
        par = 0
        for i, (nkb, live_q) in enumerate(items):
            yield from sim.wait("o_full", i & 1, ("o", i))
            for j in range(nkb):
                yield from sim.wait(f"p_full{j}", (par >> j) & 1, ("p", i))
            par ^= (1 << nkb) - 1
            if live_q[quad]:
                assert (i, 0, quad) in st["xsum"] and (nkb < 2 or (i, 1, quad) in st["xsum"])
            assert st["item"] == i, "O overwritten before the output warps read it"
            yield
            sim.bars["o_empty"].arrive(("e", i))
            if sim.bars["o_empty"].arrived == 0:
                st["o_read"] = i

    sim.run([producer(), mma()] + [softmax(h, q) for h in (0, 1) for q in range(4)] + [output(q) for q in range(4)])


def _long_items(rnd):
    items = []
    for _ in range(rnd.randint(0, 10)):
        L = rnd.choice([rnd.randint(1, 128), rnd.randint(129, 512)])
        qb = rnd.randint(0, (L - 1) // 128)
        items.append(((L + 127) // 128, [qb * 128 + q * 32 < L for q in range(4)]))
    return items


@pytest.mark.parametrize("seed", range(60))
def test_short_kernel_protocol(seed):
    short_kernel(random.Random(seed).randint(0, 14), seed)


@pytest.mark.parametrize("seed", range(60))
def test_long_kernel_protocol(seed):
    long_kernel(_long_items(random.Random(1000 + seed)), seed)


def test_planted_mistakes_are_caught():
    """Reusing a V stage one item early, or issuing S before the previous O was
    read, must trip the checks for some schedule."""
    def fails(fn):
        for seed in range(300):
            try:
                fn(seed)
            except AssertionError:
                return True
        return False

    assert fails(lambda s: short_kernel(12, s, planted=True))
    assert fails(lambda s: short_kernel(12, s, planted="s_early"))
    assert fails(lambda s: long_kernel([(4, [True] * 4)] * 6, s, planted=True))
