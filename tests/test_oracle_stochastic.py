"""Pins for the oracle's stochastic tree verification (CPU only).

Multi-step speculative sampling (SpecInfer explainer, "ツリー検証アルゴリズム":
accept a child x with probability min(1, P_LLM(x)/P_SSM(x)), otherwise
resample from norm(max(0, P_LLM - P_SSM)); the page states that the output
then follows the LLM's distribution exactly).  The oracle is treated as a
black box and pinned by that property:

* exact enumeration: for a vocab-16 (and vocab-6) toy, every tuple of child
  tokens is enumerated, the acceptance probability of each child and the
  distribution of the final draw are measured by bisecting the oracle's
  decisions over its uniform inputs, and the resulting probability of the
  first emitted token must equal softmax(l / T) to 1e-12;
* chi-square: 10^6 seeded trials on the vocab-16 toy must not reject
  P_LLM at alpha = 1e-3, for the first token and, on a depth-2 tree, for the
  second token given the accepted first node;
* special cases: q = p accepts the first child; a token with p(x) = 0 is
  always rejected and the draw is the inverse CDF of p (numpy searchsorted);
  with no tree the draw is the inverse CDF of softmax(l / T).
"""

import numpy as np
import pytest
import scipy.special
import scipy.stats

import oracle

ONE_MINUS = 1.0 - 2.0 ** -53
TINY = 2.0 ** -53


def _softmax(x):
    return scipy.special.softmax(np.asarray(x, np.float64), axis=-1)


def _run(logits, temperature, qprobs, q_row, tokens, parent, u_accept, u_sample):
    B = tokens.shape[0]
    return oracle.verify_stochastic(logits, temperature, qprobs, q_row, tokens, parent,
                                    np.full(B, tokens.shape[1], np.int32), u_accept, u_sample)


def _dyadic(prob, bits=20):
    """A distribution whose entries are multiples of 2^-bits summing to exactly
    1, so that the float32 values the oracle reads are the sampling weights."""
    c = np.floor(prob * 2 ** bits).astype(np.int64)
    c[np.argmax(c)] += 2 ** bits - c.sum()
    return (c / 2.0 ** bits).astype(np.float32)


def _toy(V, k, seed, temperature):
    rng = np.random.default_rng(seed)
    l = (2.0 * rng.standard_normal(V)).astype(np.float32)
    qs = np.stack([_dyadic(_softmax(l.astype(np.float64) + rng.standard_normal(V)))
                   for _ in range(k)])
    assert all(q.astype(np.float64).sum() == 1.0 for q in qs)
    return l, qs


def _exact_first_token_distribution(l, qs, temperature):
    """Probability of the first emitted token, integrating the oracle's
    decisions over its uniforms (children are leaves below the root)."""
    k, V = qs.shape
    tuples = np.array(np.meshgrid(*[np.arange(V)] * k, indexing="ij")).reshape(k, -1).T
    n = tuples.shape[0]
    weight = np.prod([qs[i, tuples[:, i]].astype(np.float64) for i in range(k)], axis=0)
    logits = np.broadcast_to(np.stack([l] + [l] * k)[None], (n, k + 1, V)).copy()
    qprobs = np.broadcast_to(qs[None], (n, k, V)).copy()
    q_row = np.broadcast_to(np.arange(k, dtype=np.int32)[None], (n, k)).copy()
    parent = np.full((n, k), -1, np.int32)
    tokens = tuples.astype(np.int32)

    def run(ua, us):
        return _run(logits, temperature, qprobs, q_row, tokens, parent, ua, us)

    theta = np.zeros((n, k))
    for i in range(k):
        ua = np.full((n, k), ONE_MINUS)
        lo, hi = np.zeros(n), np.ones(n)
        ua[:, i] = ONE_MINUS
        acc_hi = run(ua, np.full((n, k + 1), 0.5))["out_path"][:, 0] == i
        ua[:, i] = TINY
        acc_lo = run(ua, np.full((n, k + 1), 0.5))["out_path"][:, 0] == i
        for _ in range(64):
            mid = 0.5 * (lo + hi)
            ua[:, i] = mid
            acc = run(ua, np.full((n, k + 1), 0.5))["out_path"][:, 0] == i
            lo = np.where(acc, mid, lo)
            hi = np.where(acc, hi, mid)
        theta[:, i] = np.where(acc_hi, 1.0, np.where(acc_lo, lo, 0.0))
    reach = np.ones(n)
    prob = np.zeros(V)
    for i in range(k):
        np.add.at(prob, tuples[:, i], weight * reach * theta[:, i])
        reach = reach * (1.0 - theta[:, i])
    # distribution of the draw once every child is rejected
    ua = np.full((n, k), ONE_MINUS)
    bounds = np.zeros((n, V + 1))
    bounds[:, V] = 1.0
    for y in range(V - 1):
        lo, hi = np.zeros(n), np.ones(n)
        for _ in range(64):
            mid = 0.5 * (lo + hi)
            us = np.full((n, k + 1), 0.5)
            us[:, 0] = mid
            r = run(ua, us)
            le = r["out_tokens"][:, 0] <= y
            lo = np.where(le, mid, lo)
            hi = np.where(le, hi, mid)
        bounds[:, y + 1] = lo
    draw = np.diff(bounds, axis=1)
    prob += (weight * reach) @ draw
    return prob


@pytest.mark.parametrize("V,k,temperature", [(16, 2, 1.0), (6, 3, 0.7), (16, 1, 1.3)])
def test_exact_enumeration_equals_target(V, k, temperature):
    l, qs = _toy(V, k, 7 * V + k, temperature)
    prob = _exact_first_token_distribution(l, qs, temperature)
    p = _softmax(l.astype(np.float64) / temperature)
    np.testing.assert_allclose(prob, p, rtol=0, atol=1e-12)


def _chunked_trials(n_total, chunk, fn):
    out = []
    done = 0
    seed = 0
    while done < n_total:
        m = min(chunk, n_total - done)
        out.append(fn(m, seed))
        done += m
        seed += 1
    return out


def test_chi_square_first_token():
    V, k = 16, 3
    l, qs = _toy(V, k, 99, 1.0)
    p = _softmax(l.astype(np.float64))

    def trial(m, seed):
        rng = np.random.default_rng(1234 + seed)
        tokens = np.stack([rng.choice(V, size=m, p=qs[i].astype(np.float64) /
                                      qs[i].astype(np.float64).sum()) for i in range(k)], 1)
        r = _run(np.broadcast_to(np.stack([l] * (k + 1))[None], (m, k + 1, V)).copy(), 1.0,
                 np.broadcast_to(qs[None], (m, k, V)).copy(),
                 np.broadcast_to(np.arange(k, dtype=np.int32)[None], (m, k)).copy(),
                 tokens.astype(np.int32), np.full((m, k), -1, np.int32),
                 (rng.integers(0, 2 ** 53, (m, k)) + 0.5) * 2.0 ** -53,
                 (rng.integers(0, 2 ** 53, (m, k + 1)) + 0.5) * 2.0 ** -53)
        return np.bincount(r["out_tokens"][:, 0], minlength=V)

    counts = np.sum(_chunked_trials(1_000_000, 200_000, trial), axis=0)
    stat, pval = scipy.stats.chisquare(counts, counts.sum() * p)
    assert pval > 1e-3, (stat, pval)
    # and a plausible mistake is detected: the proposal mixture is not p
    mix = qs.astype(np.float64).mean(0)
    assert scipy.stats.chisquare(counts, counts.sum() * mix / mix.sum())[1] < 1e-6


def test_chi_square_depth_two():
    # root -> {0, 3}; 0 -> {1, 2}; 3 -> {4, 5}; every node proposed by its own SSM row
    V = 16
    parent = np.array([-1, 0, 0, -1, 3, 3], np.int32)
    T = 6
    rng0 = np.random.default_rng(5)
    L = (2.0 * rng0.standard_normal((T + 1, V))).astype(np.float32)
    qs = np.stack([_dyadic(_softmax(L[parent[u] + 1].astype(np.float64) +
                                    rng0.standard_normal(V))) for u in range(T)])
    p = _softmax(L.astype(np.float64))

    def trial(m, seed):
        rng = np.random.default_rng(777 + seed)
        tokens = np.stack([rng.choice(V, size=m, p=qs[u].astype(np.float64) /
                                      qs[u].astype(np.float64).sum()) for u in range(T)], 1)
        r = _run(np.broadcast_to(L[None], (m, T + 1, V)).copy(), 1.0,
                 np.broadcast_to(qs[None], (m, T, V)).copy(),
                 np.broadcast_to(np.arange(T, dtype=np.int32)[None], (m, T)).copy(),
                 tokens.astype(np.int32), np.broadcast_to(parent[None], (m, T)).copy(),
                 (rng.integers(0, 2 ** 53, (m, T)) + 0.5) * 2.0 ** -53,
                 (rng.integers(0, 2 ** 53, (m, T + 1)) + 0.5) * 2.0 ** -53)
        first = np.bincount(r["out_tokens"][:, 0], minlength=V)
        sec = []
        for node in (0, 3):
            sel = (r["n_accepted"] >= 1) & (r["out_path"][:, 0] == node)
            sec.append(np.bincount(r["out_tokens"][sel, 1], minlength=V))
        return first, sec[0], sec[1]

    res = _chunked_trials(1_000_000, 200_000, trial)
    first = np.sum([x[0] for x in res], axis=0)
    assert scipy.stats.chisquare(first, first.sum() * p[0])[1] > 1e-3
    for j, node in enumerate((0, 3)):
        c = np.sum([x[1 + j] for x in res], axis=0)
        assert c.sum() > 10_000
        assert scipy.stats.chisquare(c, c.sum() * p[node + 1])[1] > 1e-3


def test_q_equal_p_accepts_first_child():
    V, n = 16, 2000
    rng = np.random.default_rng(3)
    l = (2.0 * rng.standard_normal(V)).astype(np.float32)
    p = _softmax(l.astype(np.float64)).astype(np.float32)
    tokens = rng.integers(0, V, (n, 2)).astype(np.int32)
    r = _run(np.broadcast_to(np.stack([l] * 3)[None], (n, 3, V)).copy(), 1.0,
             np.broadcast_to(p[None, None], (n, 1, V)).copy(), np.zeros((n, 2), np.int32),
             tokens, np.full((n, 2), -1, np.int32),
             rng.uniform(1e-9, 1 - 1e-6, (n, 2)), rng.uniform(1e-9, 1 - 1e-9, (n, 3)))
    assert (r["n_accepted"] == 1).all() and (r["out_path"][:, 0] == 0).all()
    assert (r["out_tokens"][:, 0] == tokens[:, 0]).all()


def test_zero_target_probability_always_rejected():
    V, n = 16, 5000
    rng = np.random.default_rng(4)
    l = (2.0 * rng.standard_normal(V)).astype(np.float32)
    dead = np.array([3, 7, 11])
    l[dead] = -1.0e4                     # exp underflows: p(x) == 0 exactly
    p = _softmax(l.astype(np.float64))
    assert (p[dead] == 0).all()
    q = np.zeros(V, np.float32)
    q[dead] = np.float32(1.0 / 3.0)      # the SSM only proposes impossible tokens
    tokens = rng.choice(dead, size=(n, 2)).astype(np.int32)
    us = rng.uniform(1e-9, 1 - 1e-9, (n, 3))
    r = _run(np.broadcast_to(np.stack([l] * 3)[None], (n, 3, V)).copy(), 1.0,
             np.broadcast_to(q[None, None], (n, 1, V)).copy(), np.zeros((n, 2), np.int32),
             tokens, np.full((n, 2), -1, np.int32), rng.uniform(1e-9, 1 - 1e-9, (n, 2)), us)
    assert (r["n_accepted"] == 0).all()
    want = np.searchsorted(np.cumsum(p), us[:, 0], side="right")
    ok = (r["out_tokens"][:, 0] == want) | (r["n_flagged"] > 0)
    assert ok.all()
    assert not np.isin(r["out_tokens"][:, 0], dead).any()


@pytest.mark.parametrize("temperature", [1.0, 0.5, 2.0])
def test_no_tree_draw_is_inverse_cdf(temperature):
    V, n = 37, 4000
    rng = np.random.default_rng(int(temperature * 10))
    l = (2.0 * rng.standard_normal((n, 1, V))).astype(np.float32)
    us = rng.uniform(1e-12, 1 - 1e-12, (n, 1))
    r = oracle.verify_stochastic(l, temperature, np.zeros((n, 1, V), np.float32),
                                 np.zeros((n, 0), np.int32), np.zeros((n, 0), np.int32),
                                 np.zeros((n, 0), np.int32), np.zeros(n, np.int32),
                                 np.zeros((n, 0)), us)
    p = _softmax(l[:, 0].astype(np.float64) / temperature)
    want = np.array([np.searchsorted(np.cumsum(p[i]), us[i, 0], side="right") for i in range(n)])
    ok = (r["out_tokens"][:, 0] == want) | (r["n_flagged"] > 0)
    assert ok.all() and (r["n_accepted"] == 0).all()
    assert (r["n_decisions"] == 1).all()


def test_bad_qrow_and_token_rejected():
    V = 8
    l = np.zeros((2, 2, V), np.float32)
    r = oracle.verify_stochastic(l, 1.0, np.full((2, 1, V), 1.0 / V, np.float32),
                                 np.array([[1], [0]], np.int32), np.array([[0], [9]], np.int32),
                                 np.array([[-1], [-1]], np.int32), np.array([1, 1], np.int32),
                                 np.full((2, 1), 0.5), np.full((2, 2), 0.5))
    assert r["status"].tolist() == [oracle.BAD_QROW, oracle.BAD_TOKEN]
    assert (r["n_accepted"] == -1).all()
