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
    have read it; in the long kernel, a score buffer only after its P V is issued);
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
        self.done = 0  # products known complete: a commit's arrival covers every earlier one

    def bar(self, name, count):
        self.bars[name] = Bar(name, count)

    def commit(self, name, tag, upto=0):
        self.pending.append((name, tag, upto))

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
                n, t, upto = self.pending.pop(k)
                self.done = max(self.done, upto)
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
# Per slot (the two slots of a CTA share no barrier): items of (sequence, 128-query
# block, head), keys in 64-key blocks numbered b over the slot's items.  The
# producer loads Q of item n into buffer n % 2 and the {K, V} tiles of block b into
# stage b % NKV.  The issuer issues S of blocks b and b + 1 ahead, then per block:
# P V once the softmax has written P (score buffer b % 2), S of block b + 2 into
# that buffer (after P V in its issue order), the first P V of an item only after
# the softmax warps have read the previous item's O.  After the slot's last S, one
# commit with no product stands in for the next.  Products complete in issue
# order, and a commit's arrival means every product issued before it is complete
# (Sim.done).  A rescale of O on block b waits for S of block b + 1, which follows
# P V of block b - 1.  Every softmax warp waits for every phase of s_full in order,
# so none of these parity waits is two phases off; and P of block b - 2 is
# complete before any arrival on P of block b (one barrier per score buffer).  A
# warp arrives on the first P of an item only after reading the previous O, so the
# issuer's o_empty wait is implied by its P wait (the kernel keeps it all the same).
# planted: "s_early" issues S of block b + 2 before P V of block b; "kv_early"
# loads a K/V stage without waiting for the P V of the block it held; "rescale_s0"
# rescales O after S of block b instead of b + 1; "no_sentinel" leaves out the
# commit after the slot's last S.
def long_kernel(items, seed, planted=None):
    NKV = 4
    sim = Sim(seed)
    for i in range(2):
        sim.bar(f"q_full{i}", 1)
        sim.bar(f"q_empty{i}", 1)
        sim.bar(f"s_full{i}", 1)
        sim.bar(f"p_full{i}", 4)
    for i in range(NKV):
        sim.bar(f"kv_full{i}", 1)
        sim.bar(f"kv_empty{i}", 1)
    for n, c in (("o_full", 1), ("o_empty", 4)):
        sim.bar(n, c)
    blocks = [(n, j) for n, (nkb, _) in enumerate(items) for j in range(nkb)]
    buf = {0: None, 1: None}   # score buffer -> ("s" | "p" | "pv", block)
    o = {"item": None, "read": -1}
    written = {}               # block -> warps that have finished it
    pv_seq = {}                # block -> issue number of its P V

    def producer():
        for b, (n, j) in enumerate(blocks):
            if j == 0:
                yield from sim.wait(f"q_empty{n & 1}", ((n >> 1) & 1) ^ 1)
                sim.commit(f"q_full{n & 1}", ("q", n))
            if planted != "kv_early":
                yield from sim.wait(f"kv_empty{b % NKV}", ((b // NKV) & 1) ^ 1)
            if b >= NKV:
                assert sim.bars[f"kv_empty{b % NKV}"].phase > (b - NKV) // NKV, "K/V stage reused before its P V"
            sim.commit(f"kv_full{b % NKV}", ("kv", b))
            yield

    def issuer():
        state = {"s": 0, "seq": 0, "sentinel": False}

        def issue_s():
            b = state["s"]
            n, j = blocks[b]
            if j == 0:
                yield from sim.wait(f"q_full{n & 1}", (n >> 1) & 1, ("q", n))
            yield from sim.wait(f"kv_full{b % NKV}", (b // NKV) & 1, ("kv", b))
            prev = buf[b & 1]
            assert prev is None or prev == ("pv", b - 2), ("S over a score buffer still in use", prev, b)
            buf[b & 1] = ("s", b)
            state["seq"] += 1
            sim.commit(f"s_full{b & 1}", ("s", b), state["seq"])
            if j == items[n][0] - 1:
                sim.commit(f"q_empty{n & 1}", ("q-free", n), state["seq"])
            state["s"] += 1

        for _ in range(2):
            if state["s"] < len(blocks):
                yield from issue_s()
        oph = 0
        for b, (n, j) in enumerate(blocks):
            if planted == "s_early" and state["s"] < len(blocks) and state["s"] == b + 2:
                buf[b & 1] = ("pv", b)  # pretends P V was issued
                yield from issue_s()
            yield from sim.wait(f"p_full{b & 1}", (b >> 1) & 1, ("p", b))
            assert written.get(b) == 4, ("P V before every softmax warp wrote P", b, written.get(b))
            if j == 0:
                yield from sim.wait("o_empty", oph ^ 1, ("e", n - 1) if n else None)
                oph ^= 1
                assert o["read"] == n - 1, ("O of item", n - 1, "overwritten before it was read")
                o["item"] = n
            assert buf[b & 1] == ("s", b)
            buf[b & 1] = ("pv", b)
            state["seq"] += 1
            pv_seq[b] = state["seq"]
            sim.commit(f"kv_empty{b % NKV}", ("kv-free", b), state["seq"])
            if j == items[n][0] - 1:
                sim.commit("o_full", ("o", n), state["seq"])
            yield
            if state["s"] < len(blocks):
                yield from issue_s()
            elif not state["sentinel"] and planted != "no_sentinel":
                nb = state["s"]
                sim.commit(f"s_full{nb & 1}", ("s", nb), state["seq"])
                state["sentinel"] = True

    def softmax(q):
        oph = 0
        b = 0
        for n, (nkb, live_q) in enumerate(items):
            live = live_q[q]
            for j in range(nkb):
                yield from sim.wait(f"s_full{b & 1}", (b >> 1) & 1, ("s", b))
                assert buf[b & 1] == ("s", b), ("scores gone during the softmax", buf[b & 1], b)
                if live and j > 0 and sim.rnd.random() < 0.3:  # a rescale of O
                    nb = b if planted == "rescale_s0" else b + 1
                    yield from sim.wait(f"s_full{nb & 1}", (nb >> 1) & 1, ("s", nb))
                    assert o["item"] == n and sim.done >= pv_seq.get(b - 1, 1 << 30), \
                        ("O rescaled before P V of", b - 1, "completed")
                yield
                written[b] = written.get(b, 0) + 1
                sim.bars[f"p_full{b & 1}"].arrive(("p", b))
                b += 1
            yield from sim.wait("o_full", oph, ("o", n))
            oph ^= 1
            assert o["item"] == n
            yield
            sim.bars["o_empty"].arrive(("e", n))
            if sim.bars["o_empty"].arrived == 0:
                o["read"] = n

    sim.run([producer(), issuer()] + [softmax(q) for q in range(4)])


def _long_items(rnd):
    items = []
    for _ in range(rnd.randint(0, 10)):
        L = rnd.choice([rnd.randint(1, 128), rnd.randint(129, 512)])
        qb = rnd.randint(0, (L - 1) // 128)
        items.append(((L + 63) // 64, [qb * 128 + q * 32 < L for q in range(4)]))
    return items


@pytest.mark.parametrize("seed", range(60))
def test_short_kernel_protocol(seed):
    short_kernel(random.Random(seed).randint(0, 14), seed)


@pytest.mark.parametrize("seed", range(60))
def test_long_kernel_protocol(seed):
    long_kernel(_long_items(random.Random(1000 + seed)), seed)


def test_planted_mistakes_are_caught():
    """Reusing a V stage one item early, issuing S before the previous O was read,
    S over a score buffer before its P V, reusing a K/V stage before its P V, a
    rescale of O that waits for the wrong S, or no stand-in commit after a slot's
    last S must trip the checks for some schedule."""
    def fails(fn):
        for seed in range(300):
            try:
                fn(seed)
            except AssertionError:
                return True
        return False

    assert fails(lambda s: short_kernel(12, s, planted=True))
    assert fails(lambda s: short_kernel(12, s, planted="s_early"))
    assert fails(lambda s: long_kernel([(3, [True] * 4)] * 4, s, planted="s_early"))
    assert fails(lambda s: long_kernel([(3, [True] * 4)] * 4, s, planted="kv_early"))
    # a rescale after S of its own block, or no commit after the slot's last S
    assert fails(lambda s: long_kernel([(8, [True] * 4)] * 4, s, planted="rescale_s0"))
    assert fails(lambda s: long_kernel([(3, [True] * 4)], s, planted="no_sentinel"))
