"""Pins for the oracle's ancestor mask (CPU only).

The topology-aware mask lets node u see exactly the nodes on its root path
(SpecInfer explainer, "トークンツリー構造の仕組み" and "Tree Attention のカーネル
融合" item 1).  The oracle walks parent[] upward; these tests check it
against independent characterisations: the page's merge diagram read by
hand, subtree enumeration downward from every node, and the recursive
identity mask[u] = mask[parent(u)] | {u}.
"""

import json
import os

import numpy as np
import pytest

import oracle
from workloads import gen

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _bits(mask_row, T):
    return {v for v in range(T) if (int(mask_row[v // 32]) >> (v % 32)) & 1}


def test_merge_diagram_golden():
    g = json.load(open(os.path.join(GOLDEN, "merge_diagram.json")))
    labels, parent = g["labels"], g["parent"]
    T = len(parent)
    m = oracle.tree_mask(np.array([parent], np.int32), np.array([T], np.int32), T)
    assert m["status"][0] == 0
    for u, name in enumerate(labels):
        got = {labels[v] for v in _bits(m["mask"][0, u], T)}
        assert got == set(g["ancestors_or_self"][name]), name
        assert m["depth"][0, u] == len(g["ancestors_or_self"][name])
    # children lists in ascending index = drawing order
    fc, ns = m["first_child"][0], m["next_sibling"][0]
    for name, kids in g["children"].items():
        slot = 0 if name == "Root" else 1 + labels.index(name)
        got, c = [], fc[slot]
        while c >= 0:
            got.append(labels[c])
            c = ns[c]
        assert got == kids, name
    # each leaf's ancestor set is one candidate sequence
    leaves = [labels[u] for u in range(T) if fc[1 + u] < 0]
    seqs = sorted(sorted(g["ancestors_or_self"][n]) for n in leaves)
    assert seqs == sorted(sorted(s) for s in g["candidate_sequences"])


def test_expansion_example_golden():
    g = json.load(open(os.path.join(GOLDEN, "expansion_example.json")))
    par, _ = gen.tree_expansion(g["expansion"])
    T = len(par)
    assert T == g["n_nodes"]
    m = oracle.tree_mask(np.array([par], np.int32), np.array([T], np.int32), T)
    depth = m["depth"][0]
    assert depth.max() == g["max_depth"]
    assert np.bincount(depth)[1:].tolist() == g["nodes_per_depth"]
    assert int((m["first_child"][0, 1:] < 0).sum()) == g["n_leaves"]


def _children(par):
    ch = {-1: []}
    for u, p in enumerate(par):
        ch.setdefault(u, [])
        ch[p].append(u)
    return ch


@pytest.mark.parametrize("seed", range(12))
def test_mask_vs_subtree_enumeration(seed):
    rng = np.random.default_rng(seed)
    Tmax = [5, 31, 32, 33, 64, 100, 128][seed % 7]
    B = 4
    parent = np.full((B, Tmax), -1, np.int32)
    nn = np.zeros(B, np.int32)
    for b in range(B):
        T = int(rng.integers(0, Tmax + 1))
        par, _ = gen.tree_random(T, int(rng.integers(6, 12)), int(rng.integers(3, 6)), rng)
        if seed % 2 and T:
            perm = gen.dfs_relabel(par)
            par, _ = gen._apply_perm(par, [], perm)
        parent[b, :T] = par
        nn[b] = T
    m = oracle.tree_mask(parent, nn, Tmax)
    assert (m["status"] == 0).all()
    for b in range(B):
        T = int(nn[b])
        par = parent[b, :T].tolist()
        ch = _children(par)
        # v is an ancestor-or-self of u  <=>  u is in the subtree below v
        anc = {u: set() for u in range(T)}
        for v in range(T):
            stack = [v]
            while stack:
                x = stack.pop()
                anc[x].add(v)
                stack.extend(ch[x])
        for u in range(T):
            assert _bits(m["mask"][b, u], Tmax) == anc[u]
            assert m["depth"][b, u] == len(anc[u])
            # recursive identity
            expect = np.zeros_like(m["mask"][b, u]) if par[u] < 0 else m["mask"][b, par[u]].copy()
            expect[u // 32] |= np.uint32(1 << (u % 32))
            assert (m["mask"][b, u] == expect).all()
        # padding rows are zero / -1
        assert (m["mask"][b, T:] == 0).all() and (m["depth"][b, T:] == 0).all()
        assert (m["next_sibling"][b, T:] == -1).all()
        # child lists: ascending, complete
        for p in [-1] + list(range(T)):
            got, c = [], m["first_child"][b, p + 1]
            while c >= 0:
                got.append(int(c))
                c = m["next_sibling"][b, c]
            assert got == sorted(ch.get(p, []))


@pytest.mark.parametrize("par", [
    [0],                 # self loop
    [-1, 2, -1],         # forward reference
    [-1, -2],            # out of range below
    [-1, 0, 5],          # out of range above
    [1, 0],              # cycle
])
def test_malformed_trees_rejected(par):
    T = len(par)
    m = oracle.tree_mask(np.array([par], np.int32), np.array([T], np.int32), T)
    assert m["status"][0] == oracle.BAD_TREE
    assert (m["mask"] == 0).all()


def test_n_nodes_out_of_range():
    par = np.full((2, 4), -1, np.int32)
    m = oracle.tree_mask(par, np.array([5, -1], np.int32), 4)
    assert (m["status"] == oracle.BAD_TREE).all()


def test_empty_tree():
    m = oracle.tree_mask(np.zeros((1, 3), np.int32), np.array([0], np.int32), 3)
    assert m["status"][0] == 0 and (m["mask"] == 0).all() and (m["first_child"] == -1).all()
