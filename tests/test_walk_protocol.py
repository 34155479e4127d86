"""The stochastic walk's team exchange, on the host (CPU only).

The walk's CTAs exchange their per-chunk partial sums with no grid-wide
barrier (`csrc/verify.cu`, `csrc/team_barrier.cuh`). The K CTAs of a team
do this at every exchange n = 1, 2, ...:
1. write their (value, last index) pair into slot k of buffer n & 1;
2. publish it: a release store of n into the tag of that slot;
3. lane j of warp 0 polls the tag of slot j of that buffer until it reads
   n (an acquire), then reads slot j.

Every CTA of a team makes the same exchanges, since all of them take
identical decisions from the same slots. A slot buffer is written again two
exchanges later, and only by a CTA that has passed exchange n + 1, which
every CTA enters after reading exchange n's slots. This test replays the
exchange under random interleavings: every read must see the value written
for its own exchange, and every wait must end. A one-buffer layout is the
negative control.
"""

import random

import pytest


def _run(K, nx, seed, buffers=2):
    rnd = random.Random(seed)
    slots = [[None] * K for _ in range(buffers)]
    tags = [[0] * K for _ in range(buffers)]

    def cta(k):
        for n in range(1, nx + 1):
            buf = n % buffers
            slots[buf][k] = (n, k)                    # this CTA's partial for exchange n
            yield
            tags[buf][k] = n                          # release store of the tag
            yield
            order = list(range(K))
            rnd.shuffle(order)                        # the K lanes poll concurrently
            for j in order:
                while tags[buf][j] != n:              # acquire poll of slot j's tag
                    yield
                assert slots[buf][j] == (n, j), \
                    f"CTA {k} at exchange {n} read {slots[buf][j]} from slot {j}"
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
        assert idle < 200_000, "a team exchange never completes"


@pytest.mark.parametrize("K", [1, 2, 5, 32])
def test_slots_are_read_before_they_are_reused(K):
    for seed in range(60):
        _run(K, 7, seed)


def test_one_slot_buffer_would_race():
    # With a single buffer a fast CTA overwrites its slot for exchange n + 1
    # while a slow one still reads exchange n's values.
    with pytest.raises(AssertionError):
        for seed in range(200):
            _run(4, 6, seed, buffers=1)
