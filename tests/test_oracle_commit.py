"""Pins of the oracle's accepted-path commit (CPU only).

After verification the accepted nodes' K/V rows move to the positions right
after the committed prefix (SpecInfer explainer, "Tree Attention のカーネル融合",
item 2: the tree's KV entries stay consistent with the existing KV cache; the
flatkey.ai guide's verification diagram: the accepted prefix is committed).

Two pins tie the commit to things defined elsewhere:
  - for any node t, its tree attention over the old cache (prefix + its root
    path) must equal plain decode attention -- torch's
    scaled_dot_product_attention in fp64, a library routine -- over the first
    P + n positions of the committed cache, where the committed path is t's
    root path (n = its length); a wrong offset or head breaks it;
  - with every node's K/V row an embedding of its token, the committed rows
    must follow the tokens the verifier emitted, in order (decode attention
    cannot see the order; this pin does).
"""

import numpy as np
import pytest
import torch

import oracle
from workloads import gen


def _root_path(parent_row, t):
    path = []
    u = t
    while u >= 0:
        path.append(u)
        u = int(parent_row[u])
    return path[::-1]


def _as_f64(a, like):
    """numpy array from the oracle (bf16 as raw uint16) -> float64 tensor."""
    t = torch.from_numpy(np.ascontiguousarray(a))
    if like.dtype == torch.bfloat16:
        t = t.view(torch.int16).view(torch.bfloat16)
    return t.double()


def _paths(w, rng):
    B, Tmax = w.B, w.Tmax
    out_path = np.full((B, Tmax), -7, dtype=np.int32)
    n_acc = np.zeros(B, dtype=np.int32)
    last = np.full(B, -1, dtype=np.int64)
    for b in range(B):
        T = int(w.n_nodes[b])
        if T == 0:
            continue
        t = int(rng.integers(T))
        p = _root_path(np.asarray(w.parent[b]), t)
        out_path[b, :len(p)] = p
        n_acc[b] = len(p)
        last[b] = t
    return out_path, n_acc, last


@pytest.mark.parametrize("seed,dtype", [(1, "bf16"), (2, "f32"), (3, "bf16"), (4, "bf16")])
def test_commit_then_decode_equals_tree_attention(seed, dtype):
    w = gen.random_workload(seed, B=4, Tmax=20, Hq=4, Hkv=2, D=32, P_max=40, V=8,
                            dtype=dtype, min_nodes=1, max_depth=6)
    rng = np.random.default_rng(seed)
    out_path, n_acc, last = _paths(w, rng)
    res = oracle.kv_commit(w.k_cache, w.v_cache, w.prefix_len, out_path, n_acc)
    assert (res["status"] == 0).all()
    assert (res["new_prefix"] == np.asarray(w.prefix_len) + n_acc).all()
    K = _as_f64(res["k_cache"], w.k_cache)
    V = _as_f64(res["v_cache"], w.v_cache)
    G = w.Hq // w.Hkv
    rows = [(b, int(last[b]), h) for b in range(w.B) for h in range(w.Hq)]
    ref = oracle.tree_attention_rows(w.q, w.k_cache, w.v_cache, w.prefix_len, w.n_nodes,
                                     w.parent, w.scale, rows)
    for i, (b, t, h) in enumerate(rows):
        L = int(res["new_prefix"][b])
        qv = w.q[b, t, h].double().view(1, 1, 1, -1)
        kk = K[b, h // G, :L].view(1, 1, L, -1)
        vv = V[b, h // G, :L].view(1, 1, L, -1)
        dec = torch.nn.functional.scaled_dot_product_attention(qv, kk, vv, scale=w.scale)
        np.testing.assert_allclose(dec.view(-1).numpy(), ref[i], rtol=0, atol=1e-12)


def test_rows_outside_the_committed_range_do_not_move():
    w = gen.random_workload(7, B=5, Tmax=24, Hq=2, Hkv=2, D=16, P_max=30, V=8, min_nodes=0)
    rng = np.random.default_rng(7)
    out_path, n_acc, _ = _paths(w, rng)
    n_acc[1] = -1                      # a malformed sequence is left alone
    res = oracle.kv_commit(w.k_cache, w.v_cache, w.prefix_len, out_path, n_acc)
    k0 = oracle._np(w.k_cache)
    v0 = oracle._np(w.v_cache)
    for b in range(w.B):
        P = int(w.prefix_len[b])
        n = max(int(n_acc[b]), 0)
        assert (res["k_cache"][b, :, :P] == k0[b, :, :P]).all()
        assert (res["k_cache"][b, :, P + n:] == k0[b, :, P + n:]).all()
        assert (res["v_cache"][b, :, P + n:] == v0[b, :, P + n:]).all()
    assert res["new_prefix"][1] == int(w.prefix_len[1])
    assert (res["k_cache"][1] == k0[1]).all()


def test_identity_path_is_a_no_op():
    # a chain tree whose whole path is accepted: node i already sits at P + i
    w = gen.random_workload(8, B=2, Tmax=6, Hq=2, Hkv=1, D=16, P_max=10, V=8, ragged=False,
                            max_children=1, max_depth=6)
    path = np.tile(np.arange(6, dtype=np.int32), (2, 1))
    res = oracle.kv_commit(w.k_cache, w.v_cache, w.prefix_len, path, np.array([6, 3], np.int32))
    assert (res["k_cache"] == oracle._np(w.k_cache)).all()
    assert list(res["new_prefix"]) == [int(w.prefix_len[0]) + 6, int(w.prefix_len[1]) + 3]


@pytest.mark.parametrize("path,n", [([2, 1, 0, 0], 2),      # not increasing
                                    ([0, 6, 0, 0], 2),      # node index >= Tmax
                                    ([-1, 0, 0, 0], 1),     # negative
                                    ([0, 1, 2, 3], 7)])     # longer than Tmax
def test_malformed_paths_are_flagged_and_move_nothing(path, n):
    w = gen.random_workload(9, B=1, Tmax=6, Hq=2, Hkv=1, D=16, P_max=10, V=8, ragged=False)
    p = np.full((1, 6), 0, dtype=np.int32)
    p[0, :4] = path
    res = oracle.kv_commit(w.k_cache, w.v_cache, w.prefix_len, p, np.array([n], np.int32))
    assert res["status"][0] == oracle.BAD_PATH
    assert res["new_prefix"][0] == int(w.prefix_len[0])
    assert (res["k_cache"] == oracle._np(w.k_cache)).all()


def test_path_past_the_cache_end_is_flagged():
    w = gen.random_workload(10, B=1, Tmax=6, Hq=2, Hkv=1, D=16, P_max=10, V=8, ragged=False)
    Lmax = w.k_cache.shape[2]
    pl = np.array([Lmax - 2], dtype=np.int32)          # P + 3 >= Lmax
    p = np.array([[0, 1, 3, 0, 0, 0]], dtype=np.int32)
    res = oracle.kv_commit(w.k_cache, w.v_cache, pl, p, np.array([3], np.int32))
    assert res["status"][0] == oracle.BAD_PATH


@pytest.mark.parametrize("mode", ["greedy", "stochastic"])
def test_committed_rows_follow_the_verified_tokens_in_order(mode):
    # Every tree node's K/V row is an embedding of its token, so after the
    # commit row P + i must hold the embedding of the i-th accepted token
    # that the verifier emitted (this fixes the order, which decode
    # attention alone cannot see).
    w = gen.random_workload(11, B=6, Tmax=16, Hq=2, Hkv=2, D=16, P_max=20, V=6, dtype="f32",
                            min_nodes=2, max_children=3, max_depth=6, token_mode="topk",
                            q_sigma=0.2)
    rng = np.random.default_rng(11)
    Ek = rng.standard_normal((w.V, w.Hkv, w.D)).astype(np.float32)
    Ev = rng.standard_normal((w.V, w.Hkv, w.D)).astype(np.float32)
    k = w.k_cache.clone()
    v = w.v_cache.clone()
    for b in range(w.B):
        P = int(w.prefix_len[b])
        for u in range(int(w.n_nodes[b])):
            tok = int(w.tokens[b, u])
            k[b, :, P + u] = torch.from_numpy(Ek[tok])
            v[b, :, P + u] = torch.from_numpy(Ev[tok])
    r = oracle.workload_greedy(w) if mode == "greedy" else oracle.workload_stochastic(w)
    res = oracle.kv_commit(k, v, w.prefix_len, r["out_path"], r["n_accepted"])
    assert (res["status"] == 0).all()
    assert (r["n_accepted"] > 0).any()
    for b in range(w.B):
        P, n = int(w.prefix_len[b]), int(r["n_accepted"][b])
        for i in range(n):
            tok = int(r["out_tokens"][b, i])
            assert (res["k_cache"][b, :, P + i] == Ek[tok]).all()
            assert (res["v_cache"][b, :, P + i] == Ev[tok]).all()
