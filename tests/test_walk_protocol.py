"""The stochastic walk's team exchange, on the host (CPU only).

The walk's CTAs exchange their per-chunk partial sums with no grid-wide
barrier (`csrc/verify.cu`, `csrc/team_barrier.cuh`). The K CTAs of a team
do this at every barrier n = 1, 2, ...:
1. write their (value, last index) pair into slot k of buffer (n - 1) & 1;
2. add 1 to the team's arrival counter (a release);
3. poll until the counter reaches n·K (an acquire);
4. read all K slots of that buffer.

Every CTA of a team takes the same number of barriers, since all of them
take identical decisions from the same slots. A slot buffer is written
again two barriers later, and only by a CTA that has passed barrier n + 1,
which every CTA reaches after reading barrier n's slots. This test replays
the exchange under random interleavings: every read must see the value
written for its own barrier, and every wait must end. A one-buffer layout
is the negative control. The cluster form of the same exchange (partials
stored into every peer's shared memory, one mbarrier per buffer in every
CTA) is replayed the same way.
"""

import random

import pytest


def _run(K, nbar, seed, buffers=2):
    rnd = random.Random(seed)
    slots = [[None] * K for _ in range(buffers)]
    counter = [0]

    def cta(k):
        for n in range(1, nbar + 1):
            buf = (n - 1) % buffers
            slots[buf][k] = (n, k)                    # this CTA's partial for barrier n
            yield
            counter[0] += 1                           # release-add
            yield
            while counter[0] < n * K:                 # acquire-poll
                yield
            for j in range(K):                        # warp 0 reads the K slots
                assert slots[buf][j] == (n, j), \
                    f"CTA {k} at barrier {n} read {slots[buf][j]} from slot {j}"
                if rnd.random() < 0.3:
                    yield                             # reads spread over time

    ctas = [cta(k) for k in range(K)]
    idle = 0
    while ctas:
        i = rnd.randrange(len(ctas))
        try:
            next(ctas[i])
        except StopIteration:
            ctas.pop(i)
        idle += 1
        assert idle < 200_000, "a team barrier never completes"


@pytest.mark.parametrize("K", [1, 2, 5, 32])
def test_slots_are_read_before_they_are_reused(K):
    for seed in range(60):
        _run(K, 7, seed)


def test_one_slot_buffer_would_race():
    # With a single buffer a fast CTA overwrites its slot for barrier n + 1
    # while a slow one still reads barrier n's values.
    with pytest.raises(AssertionError):
        for seed in range(200):
            _run(4, 6, seed, buffers=1)


def _run_cluster(K, nbar, seed, buffers=2):
    """The cluster form (`csrc/cluster_xchg.cuh`): every CTA holds its own
    slots[buffers][K] and mbarriers bar[buffers] (K arrivals per phase).  At
    exchange n CTA k stores its partial into slot [n % buffers][k] of every
    CTA and arrives on every CTA's bar[n % buffers]; then it waits on its own
    barrier for phase n // buffers (by parity) and reads its own K slots."""
    rnd = random.Random(seed)
    slots = [[[None] * K for _ in range(buffers)] for _ in range(K)]   # [cta][buf][k]
    done = [[0] * buffers for _ in range(K)]        # completed phases per barrier
    pending = [[0] * buffers for _ in range(K)]     # arrivals in the open phase

    def arrive(t, buf):
        pending[t][buf] += 1
        if pending[t][buf] == K:
            pending[t][buf] = 0
            done[t][buf] += 1

    def cta(k):
        for n in range(nbar):
            buf = n % buffers
            phase = n // buffers
            for t in rnd.sample(range(K), K):          # threads 0..K-1, any order
                slots[t][buf][k] = (n, k)              # remote store, then
                arrive(t, buf)                         # remote release-arrive
                yield
            while (done[k][buf] & 1) == (phase & 1):   # parity wait (acquire)
                yield
            assert done[k][buf] == phase + 1, \
                f"CTA {k} passed exchange {n} at {done[k][buf]} completions"
            for j in range(K):
                assert slots[k][buf][j] == (n, j), \
                    f"CTA {k} at exchange {n} read {slots[k][buf][j]} from slot {j}"
                if rnd.random() < 0.3:
                    yield

    ctas = [cta(k) for k in range(K)]
    idle = 0
    while ctas:
        i = rnd.randrange(len(ctas))
        try:
            next(ctas[i])
        except StopIteration:
            ctas.pop(i)
        idle += 1
        assert idle < 200_000, "a cluster exchange never completes"


@pytest.mark.parametrize("K", [1, 2, 5, 8, 16])
def test_cluster_slots_are_read_before_they_are_reused(K):
    for seed in range(60):
        _run_cluster(K, 9, seed)


def test_cluster_one_slot_buffer_would_race():
    with pytest.raises(AssertionError):
        for seed in range(200):
            _run_cluster(4, 6, seed, buffers=1)
