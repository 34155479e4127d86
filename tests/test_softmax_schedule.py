"""The rows kernels' lazy online softmax, emulated on the host (CPU only).

For each query row the tcgen05 rows kernel processes one key tile at a
time:
1. It writes P = 2^(s·scale·log2e − m_run) against the running max m_run
   without looking at the tile's own maximum.
2. It takes the tile max (and rescales O and l) only when the tile's P sum
   exceeds 2^64 or is not finite, or when there is no running max yet.
3. Within that redo it raises m_run only when the tile max exceeds it by
   more than 8 (log2 units), so P stays below 2^8 after a redo.
P goes to the tensor cores as bf16; O and l accumulate in fp32.

This test replays that schedule in numpy (float32 accumulation, bf16
rounding of P). It checks two things against the fp64 softmax on score
sequences chosen to stress it:
- the result stays within the bf16 attention tolerance;
- no intermediate leaves the fp32 range.
It pins the design of the schedule (thresholds, redo rule, masked tiles),
not the kernel: the GPU parity tests compare the kernel itself with the
oracle.
"""

import numpy as np
import pytest

LOG2E = 1.4426950408889634
LAZY_LIMIT = 2.0 ** 64
RESCALE_THRESHOLD = 8.0
BN = 128


def _bf16(x):
    """Round float32 values to bfloat16 (nearest, ties to even), back in f32."""
    b = np.asarray(x, np.float32).view(np.uint32).astype(np.uint64)
    b = (b + 0x7FFF + ((b >> 16) & 1)) & 0xFFFF0000
    return b.astype(np.uint32).view(np.float32)


def _schedule(s, v, scale, rescale_o=True):
    """One query row: scores s [L] (-inf = masked), values v [L][D]."""
    sl2 = np.float32(scale * LOG2E)
    m_run = np.float32(-np.inf)
    l_run = np.float32(0.0)
    o = np.zeros(v.shape[1], np.float32)
    first = True
    for t0 in range(0, s.size, BN):
        st = s[t0:t0 + BN].astype(np.float32)
        vt = v[t0:t0 + BN].astype(np.float32)
        for pas in range(2):
            neg_m = np.float32(0.0) if m_run == -np.inf else -m_run
            with np.errstate(over="ignore", invalid="ignore"):
                p = np.exp2(st * sl2 + neg_m).astype(np.float32)
            lsum = np.float32(p.sum(dtype=np.float32))
            redo = not (lsum <= LAZY_LIMIT) or m_run == -np.inf
            if pas == 1 or not redo:
                break
            mt = np.float32(st.max() * sl2) if np.isfinite(st).any() else np.float32(-np.inf)
            need = mt > m_run + RESCALE_THRESHOLD
            m_new = mt if need else m_run
            alpha = np.float32(np.exp2(m_run - m_new)) if need else np.float32(1.0)
            if need and not first and rescale_o:
                o *= alpha
            l_run *= alpha
            m_run = m_new
        pb = _bf16(p)
        o += (pb[:, None] * vt).sum(axis=0, dtype=np.float32)
        l_run += lsum
        assert np.isfinite(o).all() and np.isfinite(l_run), "left the fp32 range"
        first = False
    return o / l_run if l_run > 0 else o * 0


def _exact(s, v, scale):
    s64 = s.astype(np.float64) * scale
    keep = np.isfinite(s64)
    w = np.zeros_like(s64)
    w[keep] = np.exp(s64[keep] - s64[keep].max())
    return (w[:, None] * v.astype(np.float64)).sum(0) / w.sum()


def _v(rng, L, D=64):
    return rng.standard_normal((L, D)).astype(np.float32)


CASES = {
    # ordinary scores: q.k of N(0,1) vectors in 128 dimensions
    "random": lambda rng, L: rng.standard_normal(L) * np.sqrt(128.0),
    # scores growing along the prefix: the running max is raised tile after tile
    "rising": lambda rng, L: np.linspace(-200.0, 600.0, L) + rng.standard_normal(L) * 5,
    # a huge key late in the sequence
    "late_spike": lambda rng, L: np.where(np.arange(L) == L - 7, 2000.0,
                                          rng.standard_normal(L) * 10),
    # a huge first tile, then ordinary keys that barely count
    "early_spike": lambda rng, L: np.where(np.arange(L) < 3, 1500.0, rng.standard_normal(L)),
    # scores falling along the prefix: P of later tiles underflows to 0
    "falling": lambda rng, L: np.linspace(400.0, -400.0, L),
    # the first tiles fully masked (keys outside the row's path)
    "masked_start": lambda rng, L: np.where(np.arange(L) < 2 * BN + 5, -np.inf,
                                            rng.standard_normal(L) * 20),
}


@pytest.mark.parametrize("case", sorted(CASES))
@pytest.mark.parametrize("L", [1, 129, 700, 4160])
def test_lazy_schedule_matches_softmax(case, L):
    rng = np.random.default_rng(L)
    s = np.asarray(CASES[case](rng, L), np.float64)
    if not np.isfinite(s).any():
        pytest.skip("every key masked")
    v = _v(rng, L)
    scale = 1.0 / np.sqrt(128.0)
    got = _schedule(s.astype(np.float32), v, scale)
    want = _exact(s, v, scale)
    # bf16 P (8 significant bits) against an fp64 reference, before the
    # bf16 rounding of the output: within 1e-2 of max |v|
    assert np.abs(got - want).max() <= 1e-2 * np.abs(v).max(), (case, L)


def test_without_the_redo_the_first_tile_overflows():
    # the redo rule is what keeps P finite: P against m_run = 0 on a tile of
    # scores near 1500·sqrt(128) overflows fp32
    s = np.full(BN, 1500.0 * np.sqrt(128.0), np.float32)
    sl2 = np.float32(LOG2E / np.sqrt(128.0))
    with np.errstate(over="ignore"):
        assert not np.isfinite(np.exp2(s * sl2)).all()
    got = _schedule(s, _v(np.random.default_rng(0), BN), 1.0 / np.sqrt(128.0))
    assert np.isfinite(got).all()


def test_the_check_sees_a_missing_rescale():
    # dropping the rescale of O when the running max is raised must fail
    rng = np.random.default_rng(700)
    s = np.asarray(CASES["rising"](rng, 700), np.float64)
    v = _v(rng, 700)
    got = _schedule(s.astype(np.float32), v, 1.0 / np.sqrt(128.0), rescale_o=False)
    want = _exact(s, v, 1.0 / np.sqrt(128.0))
    assert np.abs(got - want).max() > 1e-2 * np.abs(v).max()
