"""The mbarrier protocols of the tcgen05 attention kernels, on the host (CPU only).

The kernel's three roles meet only at mbarriers:
- the TMA producer fills a K ring and a V ring;
- the MMA issuer runs QK_0 .. QK_{NS-1}, then PV_j, QK_{j+NS} for each key
  tile j, committing each product to barriers;
- four softmax warps consume the scores, publish P, sometimes wait for the
  previous PV product (to rescale O), and wait for the last one before
  writing O.

This test replays exactly that sequence of arrivals and parity waits
(`csrc/attention_umma.cu`, both tile geometries) under random interleavings
of the roles, the TMA copies and the in-order tensor pipe. It checks three
things:
- no wait is left waiting for ever;
- every wait that passes sees exactly the phase it names: an mbarrier wait
  on parity p passes whenever the barrier's completed-phase count has the
  other parity, so a stale or an early pass would go unnoticed on the GPU;
- no S buffer is overwritten by a QK product before the PV product that
  reads its P has run.
"""

import random

import pytest


class _Barrier:
    def __init__(self, count):
        self.count, self.pending, self.done = count, 0, 0

    def arrive(self):
        self.pending += 1
        if self.pending == self.count:
            self.pending, self.done = 0, self.done + 1


def _run(NS, NSK, NSV, ntiles, seed, rescale_p=0.3, final_wait="o_ready", merged=True, sw=1,
         redo_p=0.2):
    """merged: the producer reuses a K slot once s_full of the QK that read it
    completes and a V slot once o_ready of the PV that read it completes (the
    rows kernels; the MMA thread then commits only to s_full and o_ready).
    sw = 2: two softmax warps per TMEM lane quarter, each on half of every
    key tile; per tile they exchange their redo votes and, when either voted,
    their row maxima (then both may rescale O), and at the end their row
    sums -- each exchange a phase of the quarter's pair mbarrier.
    The MMA model checks that the tiles it reads have landed."""
    rnd = random.Random(seed)
    nsm = 4 * sw
    bars = {"q_full": _Barrier(nsm)}
    for s in range(NSK):
        bars["k_full", s], bars["k_empty", s] = _Barrier(1), _Barrier(1)
    for s in range(NSV):
        bars["v_full", s], bars["v_empty", s] = _Barrier(1), _Barrier(1)
    for i in range(NS):
        bars["s_full", i], bars["o_ready", i] = _Barrier(1), _Barrier(1)
        bars["p_full", i] = _Barrier(nsm)
    for q in range(4):
        bars["pair", q] = _Barrier(2)
    decide = {}   # (quarter, tile) -> (redo, rescale): the same for both warps of a pair

    def shared(q, j):
        if (q, j) not in decide:
            redo = j == 0 or rnd.random() < redo_p
            decide[q, j] = (redo, redo and j > 0 and rnd.random() < rescale_p)
        return decide[q, j]

    def passes(name, k):
        """Wait for phase k of `name` (parity k & 1): True once it passes."""
        b = bars[name]
        if (b.done & 1) == (k & 1):
            return False
        assert b.done == k + 1, f"wait on {name} for phase {k} passed at {b.done} completions"
        return True

    def test(name, k):
        """A non-blocking test of phase k, issued ahead of the wait that
        reads it: the phase before k must be complete (else a stale phase
        would pass), and the result stands until it is read."""
        assert bars[name].done >= k, f"early test of {name} phase {k} at {bars[name].done}"
        return passes(name, k)

    tma, pipe = [], []
    landed = set()    # ("k" | "v", tile) whose copy has completed
    s_owner = {}       # S buffer -> tile whose scores/P it holds
    pv_done = set()

    k_read, v_read = {}, {}   # ring slot -> tile loaded there

    def pv_passed(r):
        """The wait for "PV_r done" under the commit scheme."""
        return passes(("o_ready", r % NS), r // NS)

    qk_done, pv_done_set = set(), set()

    def producer():
        # K_0 .. K_{NSK-1}, V_0 .. V_{NSV-1}, then V_m, K_{m+L} with L = NSK + NS - NSV
        lead = NSK + NS - NSV
        i = j = 0
        while i < ntiles or j < ntiles:
            if i < ntiles and (j >= ntiles or i < NSK or (j >= NSV and i <= j - 1 + lead)):
                s = i % NSK
                if i >= NSK:
                    if merged:   # QK_{i-NSK} done: s_full[i % NS], NS == NSK
                        assert NS == NSK
                        while not passes(("s_full", s), i // NS - 1):
                            yield
                    else:
                        while not passes(("k_empty", s), i // NSK - 1):
                            yield
                    assert k_read[s] in qk_done, f"K slot {s} reloaded before its QK ran"
                k_read[s] = i
                tma.append((("k_full", s), ("k", i)))
                i += 1
            else:
                s = j % NSV
                if j >= NSV:
                    if merged:   # PV_{j-NSV} done: o_ready[(j - NSV) % NS]
                        r = j - NSV
                        while not pv_passed(r):
                            yield
                    else:
                        while not passes(("v_empty", s), j // NSV - 1):
                            yield
                    assert v_read[s] in pv_done, f"V slot {s} reloaded before its PV ran"
                v_read[s] = j
                tma.append((("v_full", s), ("v", j)))
                j += 1
            yield

    def mma():
        while not passes("q_full", 0):
            yield

        def qk(i, tested=False):
            if not tested:
                while not passes(("k_full", i % NSK), i // NSK):
                    yield
            assert ("k", i) in landed, f"QK_{i} issued before K_{i} landed"
            buf = i % NS
            prev = s_owner.get(buf)
            assert prev is None or prev in pv_done or ("pv", prev) in [p[0] for p in pipe], \
                f"QK_{i} issued over the P of tile {prev} before its PV"
            commits = [("s_full", buf)] if merged else [("s_full", buf), ("k_empty", i % NSK)]
            pipe.append((("qk", i), commits))
            s_owner[buf] = i
        for i in range(min(NS, ntiles)):
            yield from qk(i)
        # V_{j+1} and K_{j+NS} are tested while the products before them are
        # issued, and waited for only when the test failed
        v_t = test(("v_full", 0), 0) if ntiles else True
        for j in range(ntiles):
            while not passes(("p_full", j % NS), j // NS):
                yield
            if not v_t:
                while not passes(("v_full", j % NSV), j // NSV):
                    yield
            assert ("v", j) in landed, f"PV_{j} issued before V_{j} landed"
            i = j + NS
            k_t = test(("k_full", i % NSK), i // NSK) if i < ntiles else True
            yield
            commits = [("o_ready", j % NS)] if merged else \
                [("v_empty", j % NSV), ("o_ready", j % NS)]
            pipe.append((("pv", j), commits))
            yield
            if i < ntiles and not k_t:
                while not passes(("k_full", i % NSK), i // NSK):
                    yield
            v_t = test(("v_full", (j + 1) % NSV), (j + 1) // NSV) if j + 1 < ntiles else True
            yield
            if i < ntiles:
                yield from qk(i, tested=True)
            yield

    def exchange(q, n):
        """Exchange n of quarter q's pair: arrive, then wait for phase n."""
        bars["pair", q].arrive()
        while not passes(("pair", q), n):
            yield

    def softmax(q):
        bars["q_full"].arrive()
        yield
        nx = 0
        s_t = test(("s_full", 0), 0) if ntiles else True
        for j in range(ntiles):
            if not s_t:
                while not passes(("s_full", j % NS), j // NS):
                    yield
            s_t = test(("s_full", (j + 1) % NS), (j + 1) // NS) if j + 1 < ntiles else True
            yield
            if sw == 1:
                rescale = j > 0 and rnd.random() < rescale_p
            else:
                redo, rescale = shared(q, j)
                yield from exchange(q, nx)              # the votes
                nx += 1
                if redo:
                    yield from exchange(q, nx)          # the row maxima
                    nx += 1
            if rescale:                                 # O rescaled: PV_{j-1} done
                while not pv_passed(j - 1):
                    yield
                assert j - 1 in pv_done
            bars["p_full", j % NS].arrive()
            yield
        if ntiles:
            last = ntiles - 1
            if final_wait == "o_ready":
                while not pv_passed(last):
                    yield
            else:                                        # the V ring's barrier instead
                while not passes(("v_empty", last % NSV), last // NSV):
                    yield
            assert set(range(ntiles)) <= pv_done
            if sw == 2:
                yield from exchange(q, nx)              # the row sums

    roles = [producer(), mma()] + [softmax(q) for q in range(4) for _ in range(sw)]
    idle = 0
    while roles or tma or pipe:
        choices = list(range(len(roles))) + (["tma"] if tma else []) + (["pipe"] if pipe else [])
        c = rnd.choice(choices)
        if c == "tma":        # copies land in any order
            bar, what = tma.pop(rnd.randrange(len(tma)))
            landed.add(what)
            bars[bar].arrive()
            idle = 0
        elif c == "pipe":     # the tensor pipe completes in issue order
            (kind, t), commits = pipe.pop(0)
            if kind == "pv":
                pv_done.add(t)
            elif kind == "qk":
                qk_done.add(t)
            for name in commits:
                bars[name].arrive()
            idle = 0
        else:
            try:
                next(roles[c])
            except StopIteration:
                roles.pop(c)
            idle += 1
        assert idle < 50_000, "no role can make progress: a wait never ends"


@pytest.mark.parametrize("NS,NSK,NSV,sw", [(3, 3, 2, 1), (2, 2, 2, 1), (3, 3, 2, 2)],
                         ids=["128-key tiles", "64-key tiles", "128-key tiles, paired softmax"])
@pytest.mark.parametrize("ntiles", [1, 2, 3, 4, 5, 8, 17])
def test_rows_kernel_protocol(NS, NSK, NSV, sw, ntiles):
    for seed in range(150):
        _run(NS, NSK, NSV, ntiles, seed, sw=sw)


@pytest.mark.parametrize("ntiles", [1, 3, 6])
def test_rows_kernel_protocol_with_ring_commits(ntiles):
    # the producer waiting on the rings' own empty barriers (the MMA thread
    # committing every product to them as well) is equally sound
    for seed in range(100):
        _run(3, 3, 2, ntiles, seed, merged=False)


def test_the_checks_catch_a_stale_wait():
    # Waiting for the last PV product on the V ring's empty barrier instead of
    # o_ready looks equivalent (PV_j also arrives there) but is not: with two
    # V stages the phase before PV_{n-1} on that barrier is PV_{n-3}, which
    # may still be running, so the parity wait can pass one phase early.  The
    # protocol check must flag it.
    with pytest.raises(AssertionError):
        for seed in range(300):
            _run(3, 3, 2, 6, seed, final_wait="v_empty", merged=False)


def _run_keysplit(NSK, NSV, ntiles, seed, rescale_p=0.3):
    """The key-split kernel: softmax group s (4 warps) takes tiles s, s+2, ...
    with its own S_s, O_s and barriers s_full[s], p_full[s], o_ready[s]; MMA
    order QK(0) QK(1), then PV(k), QK(k+2); both groups load Q (8 arrivals)."""
    rnd = random.Random(seed)
    bars = {"q_full": _Barrier(8)}
    for s in range(NSK):
        bars["k_full", s], bars["k_empty", s] = _Barrier(1), _Barrier(1)
    for s in range(NSV):
        bars["v_full", s], bars["v_empty", s] = _Barrier(1), _Barrier(1)
    for g in range(2):
        bars["s_full", g], bars["o_ready", g] = _Barrier(1), _Barrier(1)
        bars["p_full", g] = _Barrier(4)

    def passes(name, k):
        b = bars[name]
        if (b.done & 1) == (k & 1):
            return False
        assert b.done == k + 1, f"wait on {name} for phase {k} passed at {b.done} completions"
        return True

    tma, pipe, pv_done, issued_pv = [], [], set(), set()

    def producer():   # the rows kernels' load order, QK lookahead 2
        lead = NSK + 2 - NSV
        i = j = 0
        while i < ntiles or j < ntiles:
            if i < ntiles and (j >= ntiles or i < NSK or (j >= NSV and i <= j - 1 + lead)):
                s = i % NSK
                if i >= NSK:
                    while not passes(("k_empty", s), i // NSK - 1):
                        yield
                tma.append(("k_full", s))
                i += 1
            else:
                s = j % NSV
                if j >= NSV:
                    while not passes(("v_empty", s), j // NSV - 1):
                        yield
                tma.append(("v_full", s))
                j += 1
            yield

    def mma():
        while not passes("q_full", 0):
            yield

        def qk(k):
            while not passes(("k_full", k % NSK), k // NSK):
                yield
            assert k < 2 or k - 2 in issued_pv, f"QK({k}) over S_{k & 1} before PV({k - 2})"
            pipe.append((("qk", k), [("s_full", k & 1), ("k_empty", k % NSK)]))
        yield from qk(0)
        if ntiles > 1:
            yield from qk(1)
        for k in range(ntiles):
            while not passes(("p_full", k & 1), k >> 1):
                yield
            while not passes(("v_full", k % NSV), k // NSV):
                yield
            pipe.append((("pv", k), [("v_empty", k % NSV), ("o_ready", k & 1)]))
            issued_pv.add(k)
            if k + 2 < ntiles:
                yield from qk(k + 2)
            yield

    def softmax(g):
        bars["q_full"].arrive()
        yield
        mine = (ntiles - g + 1) // 2
        for mi in range(mine):
            while not passes(("s_full", g), mi):
                yield
            yield
            if mi > 0 and rnd.random() < rescale_p:
                while not passes(("o_ready", g), mi - 1):
                    yield
                assert 2 * (mi - 1) + g in pv_done
            bars["p_full", g].arrive()
            yield
        if mine:
            while not passes(("o_ready", g), mine - 1):
                yield
            assert {2 * i + g for i in range(mine)} <= pv_done

    roles = [producer(), mma()] + [softmax(g) for g in (0, 1) for _ in range(4)]
    idle = 0
    while roles or tma or pipe:
        choices = list(range(len(roles))) + (["tma"] if tma else []) + (["pipe"] if pipe else [])
        c = rnd.choice(choices)
        if c == "tma":
            bars[tma.pop(rnd.randrange(len(tma)))].arrive()
            idle = 0
        elif c == "pipe":
            (kind, t), commits = pipe.pop(0)
            if kind == "pv":
                pv_done.add(t)
            for name in commits:
                bars[name].arrive()
            idle = 0
        else:
            try:
                next(roles[c])
            except StopIteration:
                roles.pop(c)
            idle += 1
        assert idle < 50_000, "no role can make progress: a wait never ends"


@pytest.mark.parametrize("ntiles", [1, 2, 3, 4, 5, 9, 16])
def test_keysplit_kernel_protocol(ntiles):
    for seed in range(150):
        _run_keysplit(3, 2, ntiles, seed)
