"""Models of the mbarrier protocols of the backward main kernel, the forward
kernels (two tiles per CTA, one tile per CTA, CTA pairs) and the decode
kernel (bf16 cache, e4m3 cache, e4m3 cache with the FP8 PV product), run
under random interleavings (CPU only).

Each kernel role (TMA producer, MMA issuer, softmax or P/dS warps, dQ warps)
is a generator that waits on and arrives at barriers in the order the kernel
does; tcgen05 MMAs and their commits complete in issue order on a separate
"tensor core" queue, TMA loads complete in any order.  A parity wait on
phase k is only unambiguous while the barrier has completed at most k + 1
phases: the model asserts that at every check, and that every schedule runs
to completion (no deadlock).  Barriers that receive TMA bytes also count
transactions, so the pair model checks that the peer CTA's bytes landing
before the leader announced them cannot complete a phase early.  The models follow the kernels' barrier use,
not their arithmetic; they must be kept in step with the kernels by hand.
"""
import random

import pytest


class Ambiguous(AssertionError):
    pass


class Bar:
    """An mbarrier: a phase completes when its pending arrivals reach zero
    and its transaction count (expect-tx adds, complete-tx subtracts; it may
    go negative in between) is zero."""

    def __init__(self, name, count):
        self.name, self.count, self.arr, self.done, self.tx = name, count, 0, 0, 0

    def _maybe_complete(self):
        if self.arr == self.count and self.tx == 0:
            self.arr = 0
            self.done += 1

    def arrive(self, n=1, expect_tx=0):
        self.tx += expect_tx
        self.arr += n
        assert self.arr <= self.count, f"{self.name}: too many arrivals"
        self._maybe_complete()

    def complete_tx(self, nbytes):
        self.tx -= nbytes
        self._maybe_complete()

    def test(self, k):
        """Parity wait for phase k: true once phase k completed; raises if
        the barrier is two phases ahead (a parity wait would read it as
        incomplete)."""
        if self.done >= k + 2:
            raise Ambiguous(f"{self.name}: waiting for phase {k}, {self.done} phases done")
        return self.done > k


def _run(agents, tc_queue, tma, rng, limit=200000):
    """Random scheduler: steps agents, the in-order tensor-core queue and the
    unordered TMA completions until every agent finished."""
    alive = list(range(len(agents)))
    idle = 0
    for _ in range(limit):
        if not alive and not tc_queue and not tma:
            return
        c = rng.random()
        progressed = False
        if c < 0.2 and tma:
            t = tma.pop(rng.randrange(len(tma)))
            t() if callable(t) else t.arrive()
            progressed = True
        elif c < 0.4 and tc_queue:
            op = tc_queue.pop(0)
            if op is not None:
                op()
            progressed = True
        elif alive:
            i = rng.choice(alive)
            try:
                progressed = next(agents[i]) != "blocked"
            except StopIteration:
                alive.remove(i)
                progressed = True
        idle = 0 if progressed else idle + 1
        if idle > 5000 and not tc_queue and not tma:
            raise AssertionError(f"deadlock: agents {alive} blocked")
    raise AssertionError("schedule did not finish")


def _wait(bar, k):
    while not bar.test(k):
        yield "blocked"


# ----------------------------------------------------------- backward main
def backward_model(nq, stages, split_dq_full, dq_delay, rng):
    """One CTA of the backward main kernel over nq query tiles.
    split_dq_full: one dq_full barrier per tile parity (the kernel's scheme)
    or a single one; dq_delay: extra steps the dQ warps spend per tile."""
    B = {}

    def bar(name, count=1):
        return B.setdefault(name, Bar(name, count))

    for s in range(stages):
        bar(("qdo_full", s))
        bar(("qdo_empty", s))
    for b in range(2):
        bar(("s_full", b))
        bar(("dq_full", b))
    bar("dp_full")
    bar("p_full")
    bar("dq_empty")
    bar("kd_full")
    tc, tma = [], []

    def dq_full(i):
        return bar(("dq_full", i & 1)) if split_dq_full else bar(("dq_full", 0))

    def dq_phase(i):
        return (i >> 1) if split_dq_full else i

    def producer():
        for i in range(nq):
            s = i % stages
            if i >= stages:
                yield from _wait(bar(("qdo_empty", s)), i // stages - 1)
            tma.append(bar(("qdo_full", s)))
            yield "ok"

    def mma():
        def wait_q(i):
            return _wait(bar(("qdo_full", i % stages)), i // stages)
        yield from wait_q(0)
        tc.append(lambda: bar(("s_full", 0)).arrive())
        tc.append(lambda: bar("dp_full").arrive())
        if nq > 1:
            yield from wait_q(1)
            tc.append(lambda: bar(("s_full", 1)).arrive())
        for i in range(nq):
            yield from _wait(bar("p_full"), i)
            st = i % stages
            tc.append(None)  # dV, dK, dQ MMAs
            tc.append(lambda i=i: dq_full(i).arrive())
            tc.append(lambda st=st: bar(("qdo_empty", st)).arrive())
            if i + 1 < nq:
                yield from wait_q(i + 1)
                tc.append(lambda: bar("dp_full").arrive())
            if i + 2 < nq:
                yield from _wait(bar("dq_empty"), i)
                yield from wait_q(i + 2)
                tc.append(lambda i=i: bar(("s_full", i & 1)).arrive())
        tc.append(lambda: bar("kd_full").arrive())

    def pds():
        for i in range(nq):
            yield from _wait(bar(("qdo_full", i % stages)), i // stages)
            yield from _wait(bar(("s_full", i & 1)), i >> 1)
            yield "ok"  # P phase
            yield from _wait(bar("dp_full"), i)
            yield "ok"  # dS phase
            bar("p_full").arrive()
        yield from _wait(bar("kd_full"), 0)

    def dq():
        for i in range(nq):
            yield from _wait(dq_full(i), dq_phase(i))
            bar("dq_empty").arrive()
            for _ in range(dq_delay):
                yield "ok"

    return [producer(), mma(), pds(), dq()], tc, tma


@pytest.mark.parametrize("nq", [1, 2, 3, 5, 17])
@pytest.mark.parametrize("dq_delay", [0, 3, 40])
def test_backward_protocol(nq, dq_delay):
    """The kernel's scheme (dq_full per tile parity) is unambiguous and
    deadlock-free however slow the dQ warps are."""
    rng = random.Random(nq * 1000 + dq_delay)
    for _ in range(150):
        agents, tc, tma = backward_model(nq, 3, True, dq_delay, rng)
        _run(agents, tc, tma, rng)


def test_backward_single_dq_full_is_ambiguous_when_dq_is_slow():
    """The model catches the race of a single dq_full barrier: once the dQ
    warps release tile i's TMEM, the MMA warp can complete the dQ of tiles
    i+1 and i+2 before a slow dQ warp waits for tile i+1."""
    rng = random.Random(7)
    caught = False
    for _ in range(300):
        agents, tc, tma = backward_model(8, 3, False, 40, rng)
        try:
            _run(agents, tc, tma, rng)
        except Ambiguous:
            caught = True
            break
    assert caught


# ------------------------------------------------------- two-tile forward
def forward_two_tile_model(n_half, stages, rng):
    """One CTA of the two-tile forward over n_half 64-key steps (two steps
    per 128-key K/V tile, stages K/V tile buffers)."""
    B = {}

    def bar(name, count=1):
        return B.setdefault(name, Bar(name, count))

    bar("q_full")
    for s in range(stages):
        bar(("k_full", s))
        bar(("v_full", s))
        bar(("kv_empty", s))
    for b in range(2):
        bar(("s_full", b))
        bar(("p_full", b))
    bar("o_full")
    tc, tma = [], []
    n_tiles = (n_half + 1) // 2

    def producer():
        tma.append(bar("q_full"))
        for j in range(n_tiles):
            s = j % stages
            if j >= stages:
                yield from _wait(bar(("kv_empty", s)), j // stages - 1)
            tma.append(bar(("k_full", s)))
            tma.append(bar(("v_full", s)))
            yield "ok"

    def mma():
        yield from _wait(bar("q_full"), 0)
        yield from _wait(bar(("k_full", 0)), 0)
        for b in range(2):
            tc.append(lambda b=b: bar(("s_full", b)).arrive())
        for h in range(n_half):
            j = h >> 1
            s = j % stages
            hn = h + 1
            jn = hn >> 1
            yield from _wait(bar(("v_full", s)), j // stages)
            if hn < n_half:
                yield from _wait(bar(("k_full", jn % stages)), jn // stages)
            for b in range(2):
                yield from _wait(bar(("p_full", b)), h)
                tc.append(None)  # PV_b(h)
                if hn < n_half:
                    tc.append(lambda b=b: bar(("s_full", b)).arrive())
            if (h & 1) == 1 or h == n_half - 1:
                tc.append(lambda s=s: bar(("kv_empty", s)).arrive())
        tc.append(lambda: bar("o_full").arrive())

    def softmax(b):
        for h in range(n_half):
            yield from _wait(bar(("s_full", b)), h)
            yield "ok"
            bar(("p_full", b)).arrive()
        yield from _wait(bar("o_full"), 0)

    return [producer(), mma(), softmax(0), softmax(1)], tc, tma


@pytest.mark.parametrize("n_half", [1, 2, 3, 4, 7, 20])
def test_forward_two_tile_protocol(n_half):
    rng = random.Random(n_half)
    for _ in range(200):
        agents, tc, tma = forward_two_tile_model(n_half, 2, rng)
        _run(agents, tc, tma, rng)


# ----------------------------------------------------------- pair forward
def forward_pair_model(n_half, stages, rng):
    """A cluster of two CTAs of the pair forward over n_half 64-key steps.
    The leader's q_full / k_full / v_full receive both CTAs' TMA bytes (each
    CTA loads its half; the peer's bytes may land before the leader announced
    them); the leader's p_full takes one arrival per softmax warp of either
    CTA; s_full, kv_empty and o_full exist in both CTAs and the leader commits
    to both.  Each K or V half is one transaction of HALF bytes."""
    HALF = 4096
    B = {}

    def bar(name, count=1):
        return B.setdefault(name, Bar(name, count))

    for c in range(2):
        for s in range(stages):
            bar(("kv_empty", c, s))
        for b in range(2):
            bar(("s_full", c, b))
        bar(("o_full", c))
    bar("q_full")
    for s in range(stages):
        bar(("k_full", s))
        bar(("v_full", s))
    for b in range(2):
        bar(("p_full", b), 8)
    landed = {}  # (kind, step, cta) -> the CTA's half of the step is in its shared memory
    tc, tma = [], []

    def load(kind, key, cta, nbytes):
        def land():
            landed[(kind, key, cta)] = True
            bar(kind if kind == "q_full" else (kind, key % stages)).complete_tx(nbytes)
        return land

    def producer(cta):
        if cta == 0:
            bar("q_full").arrive(expect_tx=2 * 16384)
        tma.append(load("q_full", 0, cta, 16384))
        for h in range(n_half):
            s = h % stages
            if h >= stages:
                yield from _wait(bar(("kv_empty", cta, s)), h // stages - 1)
            if cta == 0:
                bar(("k_full", s)).arrive(expect_tx=2 * HALF)
            tma.append(load("k_full", h, cta, HALF))
            if cta == 0:
                bar(("v_full", s)).arrive(expect_tx=2 * HALF)
            tma.append(load("v_full", h, cta, HALF))
            yield "ok"

    def both(name):
        def commit():
            for c in range(2):
                bar((name[0], c) + name[1:]).arrive()
        return commit

    def mma():
        yield from _wait(bar("q_full"), 0)
        assert landed.get(("q_full", 0, 0)) and landed.get(("q_full", 0, 1))
        for h in range(min(2, n_half)):
            yield from _wait(bar(("k_full", h)), 0)
            assert landed.get(("k_full", h, 0)) and landed.get(("k_full", h, 1)), f"S({h}) before K landed"
            tc.append(both(("s_full", h)))
        for h in range(n_half):
            b = h & 1
            s = h % stages
            yield from _wait(bar(("v_full", s)), h // stages)
            assert landed.get(("v_full", h, 0)) and landed.get(("v_full", h, 1)), f"PV({h}) before V landed"
            yield from _wait(bar(("p_full", b)), h >> 1)
            tc.append(None)  # PV(h)
            tc.append(both(("kv_empty", s)))
            h2 = h + 2
            if h2 < n_half:
                yield from _wait(bar(("k_full", h2 % stages)), h2 // stages)
                assert landed.get(("k_full", h2, 0)) and landed.get(("k_full", h2, 1)), f"S({h2}) before K landed"
                tc.append(both(("s_full", b)))
        tc.append(both(("o_full",)))

    def softmax(cta, wg):
        i = 0
        for hs in range(wg, n_half, 2):
            yield from _wait(bar(("s_full", cta, wg)), i)
            yield "ok"
            bar(("p_full", wg)).arrive(4)  # one arrival per warp of the warpgroup
            i += 1
        yield from _wait(bar(("o_full", cta)), 0)

    agents = [producer(0), producer(1), mma()] + [softmax(c, w) for c in range(2) for w in range(2)]
    return agents, tc, tma


@pytest.mark.parametrize("n_half", [1, 2, 3, 5, 9, 20])
def test_forward_pair_protocol(n_half):
    """Both CTAs' halves of Q, K and V have landed whenever the leader's
    barrier says so (the peer's bytes may arrive before the leader's
    expect-tx), parity waits stay unambiguous, no schedule deadlocks."""
    rng = random.Random(100 + n_half)
    for _ in range(200):
        agents, tc, tma = forward_pair_model(n_half, 4, rng)
        _run(agents, tc, tma, rng)


# -------------------------------------------------------- one-tile forward
def forward_one_tile_model(n_half, stages, rng):
    """One CTA of the one-tile forward: the tile's 64-key steps alternate
    between the two softmax warpgroups (step h to warpgroup h % 2)."""
    B = {}

    def bar(name, count=1):
        return B.setdefault(name, Bar(name, count))

    bar("q_full")
    for s in range(stages):
        bar(("k_full", s))
        bar(("v_full", s))
        bar(("kv_empty", s))
    for b in range(2):
        bar(("s_full", b))
        bar(("p_full", b))
    bar("o_full")
    tc, tma = [], []
    n_tiles = (n_half + 1) // 2

    def producer():
        tma.append(bar("q_full"))
        for j in range(n_tiles):
            s = j % stages
            if j >= stages:
                yield from _wait(bar(("kv_empty", s)), j // stages - 1)
            tma.append(bar(("k_full", s)))
            tma.append(bar(("v_full", s)))
            yield "ok"

    def mma():
        yield from _wait(bar("q_full"), 0)
        for h in range(min(2, n_half)):
            yield from _wait(bar(("k_full", 0)), 0)
            tc.append(lambda h=h: bar(("s_full", h)).arrive())
        for h in range(n_half):
            b = h & 1
            j = h >> 1
            s = j % stages
            yield from _wait(bar(("v_full", s)), j // stages)
            yield from _wait(bar(("p_full", b)), h >> 1)
            tc.append(None)  # PV(h)
            if b == 1 or h == n_half - 1:
                tc.append(lambda s=s: bar(("kv_empty", s)).arrive())
            h2 = h + 2
            if h2 < n_half:
                j2 = h2 >> 1
                yield from _wait(bar(("k_full", j2 % stages)), j2 // stages)
                tc.append(lambda b=b: bar(("s_full", b)).arrive())
        tc.append(lambda: bar("o_full").arrive())

    def softmax(b):
        for i, _ in enumerate(range(b, n_half, 2)):
            yield from _wait(bar(("s_full", b)), i)
            yield "ok"
            bar(("p_full", b)).arrive()
        yield from _wait(bar("o_full"), 0)

    return [producer(), mma(), softmax(0), softmax(1)], tc, tma


@pytest.mark.parametrize("n_half", [1, 2, 3, 4, 7, 20])
def test_forward_one_tile_protocol(n_half):
    rng = random.Random(300 + n_half)
    for _ in range(200):
        agents, tc, tma = forward_one_tile_model(n_half, 2, rng)
        _run(agents, tc, tma, rng)


# ------------------------------------------------------------------ decode
def decode_model(n, stages, mode, rng):
    """One CTA of the decode kernel over n 128-slot tiles.  mode 0: bf16
    cache; 1: e4m3 cache widened by the converter warps (K into TMEM, V into
    two fp16 tiles); 2: e4m3 cache with the FP8 PV product (K widened, V read
    as loaded).  Groups of 128 threads arrive together."""
    f8, pv8 = mode >= 1, mode == 2
    B = {}

    def bar(name, count=1):
        return B.setdefault(name, Bar(name, count))

    bar("q_full")
    bar("q_conv")
    for s in range(stages):
        bar(("k_full", s))
        bar(("k_empty", s))
        bar(("v_full", s))
        bar(("v_empty", s))
    for b in range(2):
        bar(("s_full", b))
        bar(("s_free", b))
        bar(("kt_full", b))
        bar(("pv_done", b))
        bar(("v_ready", b))
    bar("p_full")
    bar("o_full")
    tc, tma = [], []

    def producer():
        tma.append(bar("q_full"))
        for i in range(n):
            s = i % stages
            if i >= stages:
                yield from _wait(bar(("k_empty", s)), i // stages - 1)
            tma.append(bar(("k_full", s)))
            if i >= stages:
                yield from _wait(bar(("v_empty", s)), i // stages - 1)
            tma.append(bar(("v_full", s)))
            yield "ok"

    def converter():
        yield from _wait(bar("q_full"), 0)
        bar("q_conv").arrive()
        for i in range(n):
            b, s = i & 1, i % stages
            if i >= 2:
                yield from _wait(bar(("s_full", b)), (i - 2) >> 1)
            yield from _wait(bar(("k_full", s)), i // stages)
            bar(("k_empty", s)).arrive()
            bar(("kt_full", b)).arrive()
            if pv8:
                continue
            if i >= 2:
                yield from _wait(bar(("pv_done", i & 1)), (i - 2) >> 1)
            yield from _wait(bar(("v_full", s)), i // stages)
            bar(("v_empty", s)).arrive()
            bar(("v_ready", i & 1)).arrive()

    def mma():
        yield from _wait(bar("q_conv" if f8 else "q_full"), 0)
        for i in range(n + 1):
            if i < n:
                b, s = i & 1, i % stages
                if i >= 2:
                    yield from _wait(bar(("s_free", b)), (i >> 1) - 1)
                if f8:
                    yield from _wait(bar(("kt_full", b)), i >> 1)
                else:
                    yield from _wait(bar(("k_full", s)), i // stages)
                tc.append(lambda b=b: bar(("s_full", b)).arrive())
                if not f8:
                    tc.append(lambda s=s: bar(("k_empty", s)).arrive())
            if i >= 1:
                j = i - 1
                sj = j % stages
                yield from _wait(bar("p_full"), j)
                if f8 and not pv8:
                    yield from _wait(bar(("v_ready", j & 1)), j >> 1)
                else:
                    yield from _wait(bar(("v_full", sj)), j // stages)
                tc.append(lambda j=j: bar(("pv_done", j & 1)).arrive())
                if not f8 or pv8:
                    tc.append(lambda sj=sj: bar(("v_empty", sj)).arrive())
        tc.append(lambda: bar("o_full").arrive())

    def softmax():
        for i in range(n):
            b = i & 1
            yield from _wait(bar(("s_full", b)), i >> 1)
            bar(("s_free", b)).arrive()
            yield "ok"
            if i > 0:
                yield from _wait(bar(("pv_done", (i - 1) & 1)), (i - 1) >> 1)
            if (not f8 or pv8) and rng.random() < 0.5:  # a tile with empty slots: zero their V rows
                yield from _wait(bar(("v_full", i % stages)), i // stages)
            bar("p_full").arrive()
        yield from _wait(bar("o_full"), 0)

    agents = [producer(), mma(), softmax()] + ([converter()] if f8 else [])
    return agents, tc, tma


@pytest.mark.parametrize("mode", [0, 1, 2])
@pytest.mark.parametrize("n", [1, 2, 3, 6, 13])
def test_decode_protocol(mode, n):
    rng = random.Random(500 + 10 * mode + n)
    for _ in range(150):
        agents, tc, tma = decode_model(n, 2, mode, rng)
        _run(agents, tc, tma, rng)
