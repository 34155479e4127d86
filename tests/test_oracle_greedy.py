"""Pins for the oracle's greedy tree verification (CPU only).

Greedy verification accepts the longest root path whose tokens all equal the
target's argmax at their parent, then appends one target token (SpecInfer
explainer, "ツリー検証アルゴリズム"; flatkey.ai guide, verification diagram:
"accept the matching prefix, plus possibly one more target token").  Pinned
against exhaustive enumeration of every root path on tiny trees with a
4-token vocabulary (which forces duplicate sibling tokens and argmax ties),
and against the chain special case, which is ordinary speculative decoding.
"""

import numpy as np
import pytest

import oracle
from workloads import gen


def _enumerate_paths(par):
    ch = {-1: []}
    for u, p in enumerate(par):
        ch.setdefault(u, [])
        ch[p].append(u)
    paths, stack = [], [[c] for c in ch[-1]]
    while stack:
        path = stack.pop()
        paths.append(path)
        stack.extend(path + [c] for c in ch[path[-1]])
    return paths


def _exhaustive(logits, tokens, par):
    am = np.argmax(logits, axis=-1)   # numpy: first index among maxima
    best = []
    for path in _enumerate_paths(par):
        rows = [0] + [1 + v for v in path[:-1]]
        if all(tokens[v] == am[r] for v, r in zip(path, rows)):
            if len(path) > len(best) or (len(path) == len(best) and path[-1] < best[-1]):
                best = path
    bonus = am[0] if not best else am[1 + best[-1]]
    return best, [int(tokens[v]) for v in best] + [int(bonus)]


@pytest.mark.parametrize("seed", range(40))
def test_greedy_vs_exhaustive_search(seed):
    rng = np.random.default_rng(seed)
    B, Tmax, V = 6, 10, 4
    parent = np.full((B, Tmax), -1, np.int32)
    nn = np.zeros(B, np.int32)
    tokens = np.zeros((B, Tmax), np.int32)
    for b in range(B):
        T = int(rng.integers(0, Tmax + 1))
        par, _ = gen.tree_random(T, 5, 3, rng)
        parent[b, :T] = par
        nn[b] = T
        tokens[b, :T] = rng.integers(0, V, T)
    # small-integer logits force argmax ties (lowest index wins)
    logits = rng.integers(-2, 3, size=(B, Tmax + 1, V)).astype(np.float32)
    r = oracle.verify_greedy(logits, tokens, parent, nn)
    assert (r["status"] == 0).all()
    for b in range(B):
        T = int(nn[b])
        path, toks = _exhaustive(logits[b], tokens[b], parent[b, :T].tolist())
        n = int(r["n_accepted"][b])
        assert n == len(path)
        assert r["out_path"][b, :n].tolist() == path
        assert r["out_tokens"][b, :n + 1].tolist() == toks
        assert (r["out_path"][b, n:] == oracle.SENTINEL).all()
        assert (r["out_tokens"][b, n + 1:] == oracle.SENTINEL).all()


@pytest.mark.parametrize("seed", range(10))
def test_chain_is_standard_speculative_decoding(seed):
    # accept draft tokens up to the first mismatch, then emit the target's token
    rng = np.random.default_rng(1000 + seed)
    T, V = 8, 5
    par = np.arange(-1, T - 1, dtype=np.int32)[None]
    logits = rng.standard_normal((1, T + 1, V)).astype(np.float32)
    am = logits[0].argmax(-1)
    tokens = am[:T].copy()[None].astype(np.int32)
    cut = int(rng.integers(0, T + 1))
    if cut < T:
        tokens[0, cut] = (am[cut] + 1) % V
    r = oracle.verify_greedy(logits, tokens, par, np.array([T], np.int32))
    assert r["n_accepted"][0] == cut
    assert r["out_tokens"][0, :cut].tolist() == am[:cut].tolist()
    assert r["out_tokens"][0, cut] == am[cut]


def test_no_tree_emits_root_argmax():
    logits = np.array([[[0.0, 3.0, 3.0, 1.0]]], np.float32)
    r = oracle.verify_greedy(logits, np.zeros((1, 0), np.int32), np.zeros((1, 0), np.int32),
                             np.array([0], np.int32))
    assert r["n_accepted"][0] == 0 and r["out_tokens"][0, 0] == 1


def test_bad_token_rejected():
    logits = np.zeros((1, 3, 4), np.float32)
    r = oracle.verify_greedy(logits, np.array([[0, 4]], np.int32), np.array([[-1, 0]], np.int32),
                             np.array([2], np.int32))
    assert r["status"][0] == oracle.BAD_TOKEN and r["n_accepted"][0] == -1
