"""The greedy verifier's walk over matched nodes, replayed on the host (CPU
only) against the oracle.

The GPU kernel `greedy_walk_kernel` does not compute the argmax of every row
with children, as the oracle's definition reads ("the deepest node whose
whole root path matches the parents' argmaxes; lowest index on ties; the
argmax of its row as the bonus token").  It walks level by level from the
root instead: the argmax of each visited row decides which of that node's
children match, the matched children form the next level, and the last
nonempty level's lowest index is the terminal.  This test replays exactly
that walk in Python on random trees -- ragged, with duplicate sibling
tokens, with argmax ties, and with every token set to its parent row's
argmax -- and requires the oracle's tokens, path and count, and that the
walk reads no row outside {root} + {fully matched nodes}.
"""

import numpy as np
import pytest

import oracle
from workloads import gen


def _walk(logits, tokens, parent, T, pick=min):
    """The kernel's walk for one sequence: (n_accepted, path, tokens out,
    rows read).  `pick` chooses the terminal among a level's nodes (the
    kernel: the lowest index)."""
    level, terminal, bonus, depth, rows = [-1], -1, 0, 0, set()
    d = 0
    while level:
        lo = pick(level)
        nxt = []
        for f in level:
            rows.add(f)
            a = int(np.argmax(logits[f + 1]))            # lowest index on ties
            if f == lo:
                terminal, bonus, depth = f, a, d
            nxt += [c for c in range(T) if parent[c] == f and tokens[c] == a]
        level = nxt
        d += 1
    path = []
    v = terminal
    while v >= 0:
        path.append(v)
        v = int(parent[v])
    path.reverse()
    assert len(path) == depth
    return depth, path, [int(tokens[u]) for u in path] + [bonus], rows


def _fully_matched(logits, tokens, parent, T):
    ok = {-1}
    for u in range(T):                                   # parents come first
        p = int(parent[u])
        if p in ok and tokens[u] == int(np.argmax(logits[p + 1])):
            ok.add(u)
    return ok


@pytest.mark.parametrize("mode", ["sample", "topk", "match", "ties"])
@pytest.mark.parametrize("seed", range(6))
def test_walk_equals_the_definition(seed, mode):
    w = gen.random_workload(300 + seed, B=24, Tmax=40, V=12 if mode == "ties" else 300,
                            min_nodes=0, max_children=5, max_depth=9,
                            token_mode="sample" if mode in ("match", "ties") else mode,
                            q_sigma=0.3, with_attention=False)
    logits = np.asarray(w.logits, dtype=np.float32)
    tokens = np.asarray(w.tokens).copy()
    parent = np.asarray(w.parent)
    if mode == "ties":   # equal maxima in every row: the lowest index must win
        logits = np.round(logits)
    for b in range(w.B):
        T = int(w.n_nodes[b])
        if mode in ("match", "ties"):
            for u in range(T):
                tokens[b, u] = int(np.argmax(logits[b, int(parent[b, u]) + 1]))
    w.tokens[:] = torch_int(tokens)
    w.logits[:] = torch_float(logits)
    ref = oracle.workload_greedy(w)
    for b in range(w.B):
        T = int(w.n_nodes[b])
        n, path, toks, rows = _walk(logits[b], tokens[b], parent[b], T)
        assert n == int(ref["n_accepted"][b]), (b, n)
        assert path == [int(x) for x in ref["out_path"][b, :n]]
        assert toks == [int(x) for x in ref["out_tokens"][b, :n + 1]]
        assert rows == _fully_matched(logits[b], tokens[b], parent[b], T)


def torch_int(a):
    import torch
    return torch.from_numpy(np.ascontiguousarray(a)).to(torch.int32)


def torch_float(a):
    import torch
    return torch.from_numpy(np.ascontiguousarray(a)).to(torch.float32)


def test_the_walk_model_sees_a_wrong_tie_rule():
    # negative control: the same walk taking a level's highest index as the
    # terminal disagrees with the oracle on trees where every token is its
    # parent row's argmax (several equally deep matched nodes)
    w = gen.random_workload(320, B=24, Tmax=40, V=300, min_nodes=0, max_children=5,
                            max_depth=9, token_mode="sample", with_attention=False)
    logits = np.asarray(w.logits, dtype=np.float32)
    parent = np.asarray(w.parent)
    tokens = np.asarray(w.tokens).copy()
    for b in range(w.B):
        for u in range(int(w.n_nodes[b])):
            tokens[b, u] = int(np.argmax(logits[b, int(parent[b, u]) + 1]))
    w.tokens[:] = torch_int(tokens)
    ref = oracle.workload_greedy(w)
    wrong = 0
    for b in range(w.B):
        T = int(w.n_nodes[b])
        n, path, _, _ = _walk(logits[b], tokens[b], parent[b], T, pick=max)
        wrong += path != [int(x) for x in ref["out_path"][b, :n]]
    assert wrong > 0
