"""A randomised model of the hand-over protocol of the paged-prefill kernel
(csrc/pa_prefill.cuh): its roles, mbarriers (waited on by phase parity, as the
hardware does) and the asynchronous tensor-core and TMA work, with random
delays.  Test infrastructure only.

Roles, as in the kernel:
* the TMA warp loads K and V tiles into rings of KS / VS stages, refilling a
  stage once its free barrier (one arrival per issuer) has completed;
* one issuer per query tile w issues QK_w(j+1) then PV_w(j) for every KV tile
  j; S/P buffers alternate by tile parity, so QK_w(j) first waits for PV_w(j-2)
  to complete (the product overwrites the P that PV_w(j-2) reads); an issuer
  whose query tile does not reach a KV tile still arrives once on its stages;
* one softmax role per query tile waits for S_w(j), sometimes rescales O (then
  waits for PV_w(j-1)), and hands P_w(j) over; the epilogue waits for the
  last PV, then stages O in the tile's Q buffer, which every QK_w product
  must have finished reading;
* with `convert` (bf16 caches) a converter role takes every landed V tile,
  rewrites it in place as fp16 (and zeroes the rows past the context end of
  the last tile), and hands it to the issuers on its own barrier per stage;
  the issuers' PV then waits on that barrier instead of the TMA's.
The tensor pipe starts products in issue order but overlaps them: a product
may start before the previous one has completed (and so before it has read
all of its operands), which is why a product that overwrites another's
operand must wait for that one's completion; a commit arrives once every
earlier product has completed.  The model checks
that no wait ever sees a phase early (parity aliasing), that every product
finds its operands in place, and that every run ends (no deadlock).
"""
from __future__ import annotations

import random


class Bar:
    def __init__(self, name, count):
        self.name, self.count, self.pending, self.done = name, count, 0, 0

    def arrive(self):
        self.pending += 1
        if self.pending == self.count:
            self.pending = 0
            self.done += 1

    def test(self, k):
        """try_wait.parity(k & 1): true iff the barrier's current phase parity
        differs from k's; it must never answer for phase k before phase k has
        completed."""
        ok = (self.done & 1) != (k & 1)
        if ok and self.done <= k:
            raise AssertionError(f"parity aliasing: {self.name} phase {k} seen with {self.done} completed")
        return ok


def run(nt_a: int, nt_b: int, seed: int, ks: int = 3, vs: int = 3, rescale_p: float = 0.3,
        max_steps: int = 400000, convert: bool = False) -> None:
    rng = random.Random(seed)
    nts = [nt_a, nt_b]
    ntiles = nts[1] if nts[1] > 0 else nts[0]
    bars = {}

    def bar(name, count=1):
        bars[name] = Bar(name, count)

    for i in range(ks):
        bar(f"k_full{i}")
        bar(f"k_free{i}", 2)
    for i in range(vs):
        bar(f"v_full{i}")
        bar(f"v_free{i}", 2)
        bar(f"v_conv{i}")
    bar("tail")
    for w in range(2):
        for b in range(2):
            bar(f"s_full{w}{b}")
            bar(f"p_full{w}{b}")
            bar(f"o_done{w}{b}")

    t = [0]
    events = []           # (time, action): TMA completions
    pipe = []             # tensor pipe queue: ("qk"|"pv", (w, j)) or ("commit", barrier)
    next_start = [0]      # the next product may start from here (overlapping the running ones)
    running = []          # (completion time, kind, (w, j)) of products started and not yet complete
    commits = []          # (barrier, products it waits for): arrives once they have all completed
    completed = set()
    s_ready, s_read, p_ready, pv_done = set(), set(), set(), set()
    k_stage, v_stage, k_landed, v_landed = {}, {}, set(), set()
    tail_zeroed = set()
    converted = set()
    zero_tail = rng.random() < 0.5
    owner = 1 if nts[1] > 0 else 0

    def wait(name, k):
        while not bars[name].test(k):
            yield None

    def load():
        for j in range(ntiles):
            if j >= ks:
                yield from wait(f"k_free{j % ks}", j // ks - 1)
            k_stage[j % ks] = j
            events.append((t[0] + rng.randint(20, 1500), ("k", j)))
            yield None
            if j >= vs:
                yield from wait(f"v_free{j % vs}", j // vs - 1)
            v_stage[j % vs] = j
            events.append((t[0] + rng.randint(20, 1500), ("v", j)))
            yield None

    def free_arrive(ring, j, stages):
        if j >= stages:
            yield from wait(f"{ring}{j % stages}", j // stages - 1)
        bars[f"{ring}{j % stages}"].arrive()

    def issuer(w):
        ntw = nts[w]

        def qk(j):
            yield from wait(f"k_full{j % ks}", j // ks)
            if j >= 2:
                yield from wait(f"o_done{w}{j & 1}", (j - 2) >> 1)
            pipe.append(("qk", (w, j)))
            pipe.append(("commit", f"s_full{w}{j & 1}"))
            pipe.append(("commit", f"k_free{j % ks}"))
            yield None

        def pv(j):
            if convert:
                yield from wait(f"v_conv{j % vs}", j // vs)
            else:
                yield from wait(f"v_full{j % vs}", j // vs)
            if zero_tail and j == ntiles - 1 and not convert:
                if w == owner:
                    tail_zeroed.add(j)
                    bars["tail"].arrive()
                else:
                    yield from wait("tail", 0)
            yield from wait(f"p_full{w}{j & 1}", j >> 1)
            pipe.append(("pv", (w, j)))
            pipe.append(("commit", f"o_done{w}{j & 1}"))
            pipe.append(("commit", f"v_free{j % vs}"))
            yield None

        if ntw > 0:
            yield from qk(0)
        else:
            yield from free_arrive("k_free", 0, ks)
        for j in range(ntiles):
            if j + 1 < ntiles:
                if j + 1 < ntw:
                    yield from qk(j + 1)
                else:
                    yield from free_arrive("k_free", j + 1, ks)
            if j < ntw:
                yield from pv(j)
            else:
                yield from free_arrive("v_free", j, vs)

    def softmax(w):
        for j in range(nts[w]):
            yield from wait(f"s_full{w}{j & 1}", j >> 1)
            assert (w, j) in s_ready, f"S({w},{j}) read before its product ran"
            s_read.add((w, j))
            for _ in range(rng.randint(1, 40)):
                yield None
            if j > 0 and rng.random() < rescale_p:      # O rescaled: PV(j-1) must have completed
                yield from wait(f"o_done{w}{(j - 1) & 1}", (j - 1) >> 1)
                assert (w, j - 1) in pv_done
            p_ready.add((w, j))
            bars[f"p_full{w}{j & 1}"].arrive()
            yield None
        if nts[w] > 0:
            yield from wait(f"o_done{w}{(nts[w] - 1) & 1}", (nts[w] - 1) >> 1)
            assert all((w, j) in pv_done for j in range(nts[w])), "epilogue before every PV completed"
            assert all((w, j) in s_ready for j in range(nts[w])), "Q buffer reused before every QK completed"

    def converter():
        for j in range(ntiles):
            yield from wait(f"v_full{j % vs}", j // vs)
            assert v_stage[j % vs] == j and j in v_landed, f"V({j}) converted before it landed"
            for _ in range(rng.randint(1, 30)):
                yield None
            if zero_tail and j == ntiles - 1:
                tail_zeroed.add(j)
            converted.add(j)
            bars[f"v_conv{j % vs}"].arrive()
            yield None

    roles = [load(), issuer(0), issuer(1), softmax(0), softmax(1)] + ([converter()] if convert else [])
    alive = [True] * len(roles)
    steps = 0
    while any(alive):
        steps += 1
        if steps > max_steps:
            raise AssertionError("deadlock: " + ", ".join(f"{n}={b.done}" for n, b in bars.items()))
        t[0] += 1
        for ev in sorted((e for e in events if e[0] <= t[0]), key=lambda e: e[0]):
            events.remove(ev)
            kind, j = ev[1]
            (k_landed if kind == "k" else v_landed).add(j)
            bars[f"{kind}_full{j % (ks if kind == 'k' else vs)}"].arrive()
        for done in [r for r in running if r[0] <= t[0]]:
            running.remove(done)
            completed.add((done[1], done[2]))
            (s_ready if done[1] == "qk" else pv_done).add(done[2])
        while commits and commits[0][1] <= completed:     # commits arrive in issue order
            bars[commits.pop(0)[0]].arrive()
        while pipe and pipe[0][0] == "commit":            # a commit does not hold back later products
            commits.append((pipe.pop(0)[1], frozenset((r[1], r[2]) for r in running)))
        if pipe:
            kind, info = pipe[0]
            if next_start[0] <= t[0]:
                pipe.pop(0)
                dur = rng.randint(5, 60)
                next_start[0] = t[0] + rng.randint(1, dur)
                running.append((t[0] + dur, kind, info))
                w, j = info
                if kind == "qk":
                    assert k_stage[j % ks] == j and j in k_landed, f"QK({w},{j}) without its K tile"
                    # S(j) overwrites the buffer that held P(j-2)
                    assert j < 2 or ((w, j - 2) in pv_done and (w, j - 2) in s_read), \
                        f"QK({w},{j}) overwrites P({w},{j - 2}) still in use"
                else:
                    assert v_stage[j % vs] == j and j in v_landed, f"PV({w},{j}) without its V tile"
                    assert (w, j) in p_ready, f"PV({w},{j}) before P was written"
                    assert not (zero_tail and j == ntiles - 1) or j in tail_zeroed
                    assert not convert or j in converted, f"PV({w},{j}) before V({j}) was converted"
        order = list(range(len(roles)))
        rng.shuffle(order)
        for i in order:
            if alive[i]:
                try:
                    next(roles[i])
                except StopIteration:
                    alive[i] = False
    # the kernel's drain: the issuers commit once more and wait, so every
    # product and commit lands before the CTA releases its memory
    for _ in range(max_steps):
        if not pipe and not running and not commits:
            break
        t[0] += 1
        for done in [r for r in running if r[0] <= t[0]]:
            running.remove(done)
            completed.add((done[1], done[2]))
        while commits and commits[0][1] <= completed:
            bars[commits.pop(0)[0]].arrive()
        while pipe and pipe[0][0] == "commit":
            commits.append((pipe.pop(0)[1], frozenset((r[1], r[2]) for r in running)))
        if pipe:
            raise AssertionError(f"product {pipe[0]} issued after every role ended")
    assert not pipe and not running and not commits, "the pipe did not drain" 
