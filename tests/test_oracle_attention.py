"""Pins for the oracle's tree attention (CPU only).

Tree attention (SpecInfer explainer, "トークンツリー構造の仕組み", equation
Attention(Q_u, K_{S_u}, V_{S_u}) = softmax(Q_u K_{S_u}^T / sqrt(d_k)) V_{S_u})
is pinned against special cases that reduce to a library routine
(torch's scaled_dot_product_attention in fp64), a closed form, and
invariances the definition implies:

* a chain-shaped tree is ordinary causal attention over prefix + chain;
* a one-node tree is single-token decode attention over prefix + itself;
* any node equals the last row of causal attention over prefix + its
  root path, the path found by enumerating root-to-leaf sequences downward;
* P = 0, one node: the output is that node's value vector exactly;
* perturbing K/V of a non-ancestor leaves the node's output unchanged;
* renumbering the nodes in another topological order permutes the outputs.
"""

import numpy as np
import pytest
import torch
import torch.nn.functional as F

import oracle
from workloads import gen


def _sdpa(q, k, v, causal, scale):
    """q [H][Lq][D], k/v [H][Lk][D] fp64 -> [H][Lq][D]."""
    return F.scaled_dot_product_attention(q[None], k[None], v[None], is_causal=causal,
                                          scale=scale)[0]


def _as64(t):
    return t.to(torch.float64)


def _paths(par):
    """Root-first path of every node, by DFS downward from the root."""
    ch = {-1: []}
    for u, p in enumerate(par):
        ch.setdefault(u, [])
        ch[p].append(u)
    out, stack = {}, [(c, [c]) for c in ch[-1]]
    while stack:
        u, path = stack.pop()
        out[u] = path
        stack.extend((c, path + [c]) for c in ch[u])
    return out


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("G", [1, 4])
def test_chain_equals_causal_attention(dtype, G):
    T, P, Hkv, D = 7, 37, 2, 64
    w = gen.random_workload(11 + G, B=1, Tmax=T, Hq=Hkv * G, Hkv=Hkv, D=D, P_max=P,
                            dtype=dtype, ragged=False)
    # overwrite the tree with a chain
    w.parent[0] = torch.arange(-1, T - 1, dtype=torch.int32)
    got = oracle.workload_attention(w)[0]          # [T][Hq][D]
    L = P + T
    for h in range(w.Hq):
        hk = h // G
        k = _as64(w.k_cache[0, hk, :L])
        v = _as64(w.v_cache[0, hk, :L])
        # queries of the prefix positions do not matter; put the chain's at P..
        qf = torch.zeros(L, D, dtype=torch.float64)
        qf[P:] = _as64(w.q[0, :, h])
        ref = _sdpa(qf[None], k[None], v[None], True, w.scale)[0][P:]
        np.testing.assert_allclose(got[:, h], ref.numpy(), rtol=0, atol=1e-12)


def test_single_node_is_decode_attention():
    w = gen.random_workload(5, B=3, Tmax=1, Hq=8, Hkv=2, D=128, P_max=300, P_min=1,
                            dtype="bf16", ragged=False)
    got = oracle.workload_attention(w)
    for b in range(w.B):
        P = int(w.prefix_len[b])
        for h in range(w.Hq):
            hk = h // w.G
            k = _as64(w.k_cache[b, hk, :P + 1])
            v = _as64(w.v_cache[b, hk, :P + 1])
            q = _as64(w.q[b, 0, h])[None]
            ref = _sdpa(q[None], k[None], v[None], False, w.scale)[0, 0]
            np.testing.assert_allclose(got[b, 0, h], ref.numpy(), rtol=0, atol=1e-12)


def test_empty_prefix_single_node_returns_value():
    w = gen.random_workload(6, B=2, Tmax=1, Hq=4, Hkv=4, D=64, P_max=0, dtype="bf16",
                            ragged=False)
    got = oracle.workload_attention(w)
    for b in range(2):
        for h in range(4):
            assert (got[b, 0, h] == _as64(w.v_cache[b, h, 0]).numpy()).all()


@pytest.mark.parametrize("seed", range(6))
def test_every_node_is_causal_attention_over_its_path(seed):
    dtype = "f32" if seed % 2 else "bf16"
    Hkv, G = [(1, 1), (2, 4), (4, 2)][seed % 3]
    w = gen.random_workload(100 + seed, B=3, Tmax=20, Hq=Hkv * G, Hkv=Hkv, D=64, P_max=90,
                            dtype=dtype, dfs=bool(seed % 2))
    got = oracle.workload_attention(w)
    for b in range(w.B):
        T, P = int(w.n_nodes[b]), int(w.prefix_len[b])
        paths = _paths(w.parent[b, :T].tolist())
        for u in range(T):
            pos = list(range(P)) + [P + v for v in paths[u]]
            for h in range(w.Hq):
                hk = h // G
                k = _as64(w.k_cache[b, hk, pos])
                v = _as64(w.v_cache[b, hk, pos])
                qf = torch.zeros(len(pos), w.D, dtype=torch.float64)
                qf[-1] = _as64(w.q[b, u, h])
                ref = _sdpa(qf[None], k[None], v[None], True, w.scale)[0, -1]
                np.testing.assert_allclose(got[b, u, h], ref.numpy(), rtol=0, atol=1e-12)
        # padding rows untouched
        assert np.isnan(got[b, T:]).all()


def test_non_ancestor_perturbation_invariance():
    w = gen.random_workload(7, B=1, Tmax=24, Hq=4, Hkv=2, D=64, P_max=50, dtype="f32",
                            ragged=False)
    T, P = int(w.n_nodes[0]), int(w.prefix_len[0])
    base = oracle.workload_attention(w)
    m = oracle.tree_mask(w.parent, w.n_nodes, w.Tmax)["mask"][0]
    rng = np.random.default_rng(0)
    for u in range(T):
        anc = {v for v in range(T) if (int(m[u, v // 32]) >> (v % 32)) & 1}
        others = [v for v in range(T) if v not in anc]
        if not others:
            continue
        w2_k, w2_v = w.k_cache.clone(), w.v_cache.clone()
        for v in others:
            w2_k[0, :, P + v] = torch.from_numpy(rng.standard_normal((2, 64)) * 50).float()
            w2_v[0, :, P + v] = torch.from_numpy(rng.standard_normal((2, 64)) * 50).float()
        out = oracle.tree_attention(w.q, w2_k, w2_v, w.prefix_len, w.n_nodes, w.parent, w.scale)
        assert (out[0, u] == base[0, u]).all()
        # and perturbing an ancestor does change it
        v = max(anc)
        w2_k[0, :, P + v] += 1.0
        out = oracle.tree_attention(w.q, w2_k, w.v_cache, w.prefix_len, w.n_nodes, w.parent,
                                    w.scale)
        assert not (out[0, u] == base[0, u]).all()


def test_relabel_permutes_outputs():
    # creation order (random topological) vs depth-first order of one tree
    w = gen.random_workload(8, B=1, Tmax=30, Hq=4, Hkv=2, D=64, P_max=40, dtype="f32",
                            ragged=False, dfs=False)
    T, P = int(w.n_nodes[0]), int(w.prefix_len[0])
    par = w.parent[0, :T].tolist()
    perm = gen.dfs_relabel(par)              # perm[new] = old
    new_par, _ = gen._apply_perm(par, [], perm)
    q2, k2, v2 = w.q.clone(), w.k_cache.clone(), w.v_cache.clone()
    for new, old in enumerate(perm):
        q2[0, new] = w.q[0, old]
        k2[0, :, P + new] = w.k_cache[0, :, P + old]
        v2[0, :, P + new] = w.v_cache[0, :, P + old]
    p2 = w.parent.clone()
    p2[0, :T] = torch.tensor(new_par, dtype=torch.int32)
    a = oracle.workload_attention(w)
    b = oracle.tree_attention(q2, k2, v2, w.prefix_len, w.n_nodes, p2, w.scale)
    for new, old in enumerate(perm):
        np.testing.assert_allclose(b[0, new], a[0, old], rtol=0, atol=1e-13)


def test_rows_api_matches_full():
    w = gen.random_workload(9, B=2, Tmax=10, Hq=6, Hkv=3, D=64, P_max=70, dtype="bf16")
    full = oracle.workload_attention(w)
    sel = [(b, u, h) for b in range(2) for u in range(int(w.n_nodes[b])) for h in (0, 5)]
    rows = oracle.tree_attention_rows(w.q, w.k_cache, w.v_cache, w.prefix_len, w.n_nodes,
                                      w.parent, w.scale, sel)
    for i, (b, u, h) in enumerate(sel):
        assert (rows[i] == full[b, u, h]).all()


def test_malformed_tree_raises():
    w = gen.random_workload(10, B=1, Tmax=4, Hq=2, Hkv=2, D=64, P_max=10, ragged=False)
    w.parent[0, 1] = 3
    with pytest.raises(ValueError):
        oracle.workload_attention(w)
