"""Input-generator checks (CPU only): tree shapes of the five workloads and
the SplitMix64 uniform stream."""

import numpy as np
import pytest

import oracle
from workloads import gen


def _splitmix_reference(seed, n):
    # The published stateful recurrence, with Python integers.
    out, x = [], seed
    for _ in range(n):
        x = (x + 0x9E3779B97F4A7C15) & (2 ** 64 - 1)
        z = x
        z = ((z ^ (z >> 30)) * 0xBF58476D1CE4E5B9) & (2 ** 64 - 1)
        z = ((z ^ (z >> 27)) * 0x94D049BB133111EB) & (2 ** 64 - 1)
        out.append(z ^ (z >> 31))
    return out


@pytest.mark.parametrize("seed", [0, 1, 20261202, 2 ** 63 + 5])
def test_splitmix64_matches_recurrence(seed):
    got = gen._splitmix64(seed, 50).tolist()
    assert got == _splitmix_reference(seed, 50)
    u = gen.splitmix64_uniforms(seed, 100000)
    assert (u > 0).all() and (u < 1).all()
    assert abs(u.mean() - 0.5) < 0.01


def _depths(par):
    d = []
    for u, p in enumerate(par):
        d.append(1 if p < 0 else d[p] + 1)
    return d


def test_config_tree_shapes():
    w0 = gen.config_workload(0)
    assert w0.parent[0].tolist() == [-1, -1, 0, 0, 1, 1]
    w1 = gen.config_workload(1, with_attention=False)
    for b in range(w1.B):
        par = w1.parent[b].tolist()
        assert int(w1.n_nodes[b]) == 20 and max(_depths(par)) == 8
    w2 = gen.config_workload(2, with_attention=False)
    for b in range(w2.B):
        T = int(w2.n_nodes[b])
        par = w2.parent[b, :T].tolist()
        assert 8 <= T <= 24 and max(_depths(par)) == 8
        assert sum(1 for u in range(T) if u not in par) == 3      # 3 leaves: 3 chains
        # merged siblings carry distinct tokens
        for p in set(par):
            toks = [int(w2.tokens[b, u]) for u in range(T) if par[u] == p]
            assert len(toks) == len(set(toks))
    w3 = gen.config_workload(3, B=4, with_attention=False)
    for b in range(w3.B):
        par = w3.parent[b].tolist()
        assert int(w3.n_nodes[b]) == 64 and max(_depths(par)) <= 8
        assert max(np.bincount(np.array(par) + 1)) <= 5
    w4 = gen.config_workload(4, B=1, with_attention=False)
    par = w4.parent[0].tolist()
    assert int(w4.n_nodes[0]) == 128
    assert np.bincount(_depths(par))[1:].tolist() == [5, 25, 34, 32, 20, 12]


def test_trees_are_depth_first_and_valid():
    for i in (1, 2, 3):
        w = gen.config_workload(i, B=3, with_attention=False)
        m = oracle.tree_mask(w.parent, w.n_nodes, w.Tmax)
        assert (m["status"] == 0).all()
        for b in range(w.B):
            T = int(w.n_nodes[b])
            par = w.parent[b, :T].tolist()
            # pre-order: each node's subtree is a contiguous index range
            size = [1] * T
            for u in reversed(range(T)):
                if par[u] >= 0:
                    size[par[u]] += size[u]
            for u in range(T):
                for v in range(u + 1, u + size[u]):
                    bits = m["mask"][b, v]
                    assert (int(bits[u // 32]) >> (u % 32)) & 1


def test_seeded_determinism():
    a = gen.random_workload(3, B=2)
    b = gen.random_workload(3, B=2)
    for f in ("parent", "tokens", "q", "k_cache", "logits", "q_probs", "u_accept"):
        assert (getattr(a, f) == getattr(b, f)).all()
