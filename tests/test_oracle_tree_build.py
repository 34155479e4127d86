"""Pins of the oracle's token-tree construction (CPU only).

SpecInfer explainer, section "マルチドラフトモデルアプローチ": an expansion-
based tree <k_1, ..., k_n> takes one SSM's top-k_i tokens at every node of
depth i-1 (item 1, example <1,1,3,1,1,1,1,1>); a merge-based tree merges the
outputs of several SSMs into one token tree (item 2, the graph TD figure);
"Tree Attention のカーネル融合", item 2: the tree is laid out depth-first.

Pins: the page's expansion example (node and leaf counts, depth profile --
tests/golden/expansion_example.json); the page's merge figure read by hand
(tests/golden/merge_diagram.json), rebuilt from its three candidate
sequences; the top-k order against numpy's lexsort; depth-first pre-order
against a recursive walk written here; malformed inputs.
"""

import json
import os

import numpy as np
import pytest

import oracle

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _empty(B, Tmax):
    z = np.zeros((B, Tmax), dtype=np.int32)
    return z.copy(), z.copy(), z.copy(), np.zeros(B, np.int32), np.zeros(B, np.int32)


def _expand_all(ks, V=16, B=2, Tmax=64, seed=0):
    """Run the expansion level by level; frontier node i reads q row
    (its node index + 1), the root row 0 (a distinct row per node)."""
    rng = np.random.default_rng(seed)
    q = rng.random((B, Tmax + 1, V)).astype(np.float32)
    par, tok, qr, nn, lb = _empty(B, Tmax)
    for k in ks:
        frow = np.zeros((B, Tmax), dtype=np.int32)
        for b in range(B):
            if nn[b] == 0:
                frow[b, 0] = 0
            else:
                F = nn[b] - lb[b]
                frow[b, :F] = np.arange(lb[b], nn[b]) + 1
        r = oracle.tree_expand(q, frow, k, par, tok, qr, nn, lb)
        assert (r["status"] == 0).all()
        par, tok, qr, nn, lb = r["parent"], r["tokens"], r["q_row"], r["n_nodes"], r["lvl_begin"]
    return q, par, tok, qr, nn


def _depths(par, T):
    d = []
    for u in range(T):
        x, n = u, 0
        while x >= 0:
            x, n = int(par[x]), n + 1
        d.append(n)
    return d


def test_expansion_example_from_the_page():
    g = json.load(open(os.path.join(GOLDEN, "expansion_example.json")))
    _, par, tok, qr, nn = _expand_all(g["expansion"])
    for b in range(par.shape[0]):
        T = int(nn[b])
        assert T == g["n_nodes"]
        d = _depths(par[b], T)
        assert max(d) == g["max_depth"]
        assert [d.count(i + 1) for i in range(max(d))] == g["nodes_per_depth"]
        leaves = [u for u in range(T) if u not in set(par[b, :T].tolist())]
        assert len(leaves) == g["n_leaves"]


def test_children_are_the_top_k_of_their_row():
    q, par, tok, qr, nn = _expand_all((3, 2, 2), V=12, seed=3)
    for b in range(par.shape[0]):
        T = int(nn[b])
        for p in [-1] + list(range(T)):
            kids = [u for u in range(T) if par[b, u] == p]
            if not kids:
                continue
            rows = {int(qr[b, u]) for u in kids}
            assert len(rows) == 1
            row = q[b, rows.pop()].astype(np.float64)
            order = np.lexsort((np.arange(row.size), -row))   # prob desc, id asc
            assert [int(tok[b, u]) for u in kids] == order[:len(kids)].tolist()


def test_topk_ties_take_the_lower_token_id():
    B, Tmax, V = 1, 8, 6
    q = np.array([[[0.2, 0.3, 0.3, 0.1, 0.3, 0.0]]], dtype=np.float32)
    par, tok, qr, nn, lb = _empty(B, Tmax)
    r = oracle.tree_expand(q, np.zeros((B, Tmax), np.int32), 4, par, tok, qr, nn, lb)
    assert r["tokens"][0, :4].tolist() == [1, 2, 4, 0]
    assert r["parent"][0, :4].tolist() == [-1] * 4


def _preorder(par, T):
    kids = {u: [v for v in range(T) if par[v] == u] for u in range(-1, T)}
    out = []

    def walk(u):
        out.append(u)
        for v in kids[u]:
            walk(v)
    for v in kids[-1]:
        walk(v)
    return out


@pytest.mark.parametrize("seed", range(4))
def test_dfs_order_is_the_recursive_preorder(seed):
    rng = np.random.default_rng(seed)
    B, Tmax = 3, 40
    par = np.full((B, Tmax), -7, np.int32)
    tok = rng.integers(0, 100, (B, Tmax)).astype(np.int32)
    qr = rng.integers(0, 9, (B, Tmax)).astype(np.int32)
    nn = np.array([40, 1, 17], np.int32)
    for b in range(B):
        for u in range(int(nn[b])):
            par[b, u] = int(rng.integers(-1, u))   # any earlier node, or the root
    r = oracle.tree_dfs_order(par, tok, qr, nn)
    assert (r["status"] == 0).all()
    for b in range(B):
        T = int(nn[b])
        order = _preorder(par[b], T)
        assert r["perm"][b, :T].tolist() == order
        inv = {old: new for new, old in enumerate(order)}
        assert r["parent"][b, :T].tolist() == [-1 if par[b, o] < 0 else inv[int(par[b, o])]
                                               for o in order]
        assert r["tokens"][b, :T].tolist() == [int(tok[b, o]) for o in order]
        assert r["q_row"][b, :T].tolist() == [int(qr[b, o]) for o in order]
        # pre-order: every subtree is the contiguous range after its root
        for u in range(T):
            sub = [v for v in range(T) if _is_desc(r["parent"][b], v, u)]
            assert sub == list(range(u, u + len(sub)))


def _is_desc(par, v, u):
    while v >= 0:
        if v == u:
            return True
        v = int(par[v])
    return False


def test_merge_rebuilds_the_page_figure():
    g = json.load(open(os.path.join(GOLDEN, "merge_diagram.json")))
    labels = g["labels"]
    tok_id = {name: i for i, name in enumerate("ABCDEFGH")}
    seqs = g["candidate_sequences"]          # A C F / A D G / B E H
    M, L = len(seqs), max(len(s) for s in seqs)
    ct = np.zeros((1, M, L), np.int32)
    cq = np.zeros((1, M, L), np.int32)
    for m, sq in enumerate(seqs):
        ct[0, m, :len(sq)] = [tok_id[x] for x in sq]
        cq[0, m, :len(sq)] = [10 * m + i for i in range(len(sq))]
    r = oracle.tree_merge_chains(ct, cq, np.array([[len(s) for s in seqs]], np.int32), Tmax=16)
    assert r["status"][0] == 0 and r["n_nodes"][0] == len(labels)
    T = len(labels)
    assert r["parent"][0, :T].tolist() == g["parent"]
    assert ["ABCDEFGH"[t] for t in r["tokens"][0, :T]] == labels
    # the shared node A keeps the q row of the chain that created it (chain 0)
    assert r["q_row"][0, 0] == 0 and r["q_row"][0, 3] == 11   # D: chain 1, step 1


def test_merge_shares_prefixes_and_respects_capacity():
    ct = np.array([[[5, 6, 7], [5, 6, 8], [9, 0, 0]]], np.int32)
    cq = np.arange(9, dtype=np.int32).reshape(1, 3, 3)
    r = oracle.tree_merge_chains(ct, cq, np.array([[3, 3, 1]], np.int32), Tmax=8)
    assert r["n_nodes"][0] == 5                       # 5-6-7, 8 under 6, 9
    assert r["parent"][0, :5].tolist() == [-1, 0, 1, 1, -1]
    assert r["tokens"][0, :5].tolist() == [5, 6, 7, 8, 9]
    r = oracle.tree_merge_chains(ct, cq, np.array([[3, 3, 1]], np.int32), Tmax=4)
    assert r["status"][0] == 1 and r["n_nodes"][0] == -1


def test_expand_rejects_overflow_and_bad_rows():
    B, Tmax, V = 1, 4, 8
    q = np.random.default_rng(0).random((B, 2, V)).astype(np.float32)
    par, tok, qr, nn, lb = _empty(B, Tmax)
    r = oracle.tree_expand(q, np.zeros((B, Tmax), np.int32), 5, par, tok, qr, nn, lb)
    assert r["status"][0] == 1 and r["n_nodes"][0] == 0           # 5 > Tmax
    fr = np.full((B, Tmax), 7, np.int32)                          # q row out of range
    r = oracle.tree_expand(q, fr, 2, par, tok, qr, nn, lb)
    assert r["status"][0] == 1 and r["n_nodes"][0] == 0
