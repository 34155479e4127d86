"""GPU parity of token-tree construction (tsd_tree_expand, tsd_tree_dfs_order,
tsd_tree_merge_chains) against the oracle: integer outputs, bit-exact."""

import numpy as np
import pytest
import torch

import oracle
import tree_speculative_decoding_ancestor_b200 as tsd

pytestmark = pytest.mark.gpu


def _status(dev):
    torch.cuda.synchronize(dev)
    return int(tsd.device_status(dev).item())


def _q(seed, B, R, V, ties):
    rng = np.random.default_rng(seed)
    q = rng.random((B, R, V)).astype(np.float32)
    if ties:   # coarse values: many exact ties
        q = (np.floor(q * 8) / 8).astype(np.float32)
    return q


# k <= 8 takes the one-pass register top-k (lists of 2, 4 or 8 per thread),
# k > 8 one block pass per child; V % 4 != 0 takes the scalar loads.
@pytest.mark.parametrize("ks,V,ties", [((2, 3, 2), 1000, False), ((1, 1, 3, 1, 1, 1, 1, 1), 32000, False),
                                       ((4, 2), 37, True), ((5, 5, 2), 128256, False),
                                       ((8, 2), 600, True), ((9, 3), 1000, True),
                                       ((7, 6), 1001, False), ((16,), 40, True)])
def test_expansion_matches_oracle(cuda_device, ks, V, ties):
    B, Tmax = 3, 128
    dev = cuda_device
    q = _q(len(ks) + V, B, Tmax + 1, V, ties)
    z = np.zeros((B, Tmax), np.int32)
    o_par, o_tok, o_qr = z.copy(), z.copy(), z.copy()
    o_nn, o_lb = np.zeros(B, np.int32), np.zeros(B, np.int32)
    tree = tsd.Tree(*(torch.zeros((B, Tmax), dtype=torch.int32, device=dev) for _ in range(3)),
                    torch.zeros(B, dtype=torch.int32, device=dev))
    lb = torch.zeros(B, dtype=torch.int32, device=dev)
    qd = torch.from_numpy(q).to(dev)
    tsd.device_status(dev).zero_()
    for k in ks:
        frow = np.zeros((B, Tmax), np.int32)
        for b in range(B):
            if o_nn[b] > 0:
                F = o_nn[b] - o_lb[b]
                frow[b, :F] = np.arange(o_lb[b], o_nn[b]) + 1   # node u's row is u + 1
        r = oracle.tree_expand(q, frow, k, o_par, o_tok, o_qr, o_nn, o_lb)
        assert (r["status"] == 0).all()
        o_par, o_tok, o_qr, o_nn, o_lb = (r["parent"], r["tokens"], r["q_row"], r["n_nodes"],
                                          r["lvl_begin"])
        tsd.tree_expand(qd, torch.from_numpy(frow).to(dev), k, tree, lb)
    assert _status(dev) == 0
    assert (tree.n_nodes.cpu().numpy() == o_nn).all()
    assert (lb.cpu().numpy() == o_lb).all()
    for b in range(B):
        T = int(o_nn[b])
        assert (tree.parent[b, :T].cpu().numpy() == o_par[b, :T]).all()
        assert (tree.tokens[b, :T].cpu().numpy() == o_tok[b, :T]).all()
        assert (tree.q_row[b, :T].cpu().numpy() == o_qr[b, :T]).all()
    # depth-first renumbering of the expanded trees
    perm, dfs = tsd.tree_dfs_order(tree)
    r = oracle.tree_dfs_order(o_par, o_tok, o_qr, o_nn)
    for b in range(B):
        T = int(o_nn[b])
        assert (perm[b, :T].cpu().numpy() == r["perm"][b, :T]).all()
        assert (dfs.parent[b, :T].cpu().numpy() == r["parent"][b, :T]).all()
        assert (dfs.tokens[b, :T].cpu().numpy() == r["tokens"][b, :T]).all()
        assert (dfs.q_row[b, :T].cpu().numpy() == r["q_row"][b, :T]).all()


def test_expansion_overflow_is_flagged(cuda_device):
    dev = cuda_device
    B, Tmax, V = 2, 8, 50
    q = torch.rand((B, 4, V), device=dev)
    tree = tsd.Tree(*(torch.zeros((B, Tmax), dtype=torch.int32, device=dev) for _ in range(3)),
                    torch.zeros(B, dtype=torch.int32, device=dev))
    lb = torch.zeros(B, dtype=torch.int32, device=dev)
    tsd.device_status(dev).zero_()
    frow = torch.zeros((B, Tmax), dtype=torch.int32, device=dev)
    tsd.tree_expand(q, frow, 5, tree, lb)                 # root -> 5 nodes: fits
    assert _status(dev) == 0
    frow[:, :5] = torch.arange(1, 4, device=dev).repeat(2)[:5]
    tsd.tree_expand(q, frow, 2, tree, lb)                 # 5 + 10 > 8: refused on the device
    assert _status(dev) & tsd.binding.DEV_BAD_TREE
    assert (tree.n_nodes == 5).all().item() and (lb == 0).all().item()
    tsd.device_status(dev).zero_()
    with pytest.raises(tsd.TsdError):                     # k > Tmax: refused on the host
        tsd.tree_expand(q, frow, 9, tree, lb)


@pytest.mark.parametrize("seed", [1, 2, 3])
def test_dfs_order_of_random_trees(cuda_device, seed):
    rng = np.random.default_rng(seed)
    B, Tmax = 16, 128
    par = np.full((B, Tmax), -1, np.int32)
    nn = rng.integers(0, Tmax + 1, B).astype(np.int32)
    for b in range(B):
        for u in range(int(nn[b])):
            par[b, u] = int(rng.integers(-1, u))
    tok = rng.integers(0, 999, (B, Tmax)).astype(np.int32)
    qr = rng.integers(0, 50, (B, Tmax)).astype(np.int32)
    dev = cuda_device
    t = tsd.Tree(*(torch.from_numpy(a).to(dev) for a in (par, tok, qr, nn)))
    perm, dfs = tsd.tree_dfs_order(t)
    assert _status(dev) == 0
    r = oracle.tree_dfs_order(par, tok, qr, nn)
    for b in range(B):
        T = int(nn[b])
        assert (perm[b, :T].cpu().numpy() == r["perm"][b, :T]).all()
        assert (dfs.parent[b, :T].cpu().numpy() == r["parent"][b, :T]).all()
        assert (dfs.tokens[b, :T].cpu().numpy() == r["tokens"][b, :T]).all()


@pytest.mark.parametrize("seed,M,L,V", [(5, 3, 8, 6), (6, 8, 16, 3), (7, 4, 32, 2)])
def test_merge_matches_oracle(cuda_device, seed, M, L, V):
    rng = np.random.default_rng(seed)
    B = 12
    ct = rng.integers(0, V, (B, M, L)).astype(np.int32)   # a small vocabulary forces sharing
    for b in range(B):
        for m in range(1, M):   # chains copying a prefix of an earlier chain
            s = int(rng.integers(0, L))
            ct[b, m, :s] = ct[b, int(rng.integers(0, m)), :s]
    cq = rng.integers(0, 99, (B, M, L)).astype(np.int32)
    cl = rng.integers(0, L + 1, (B, M)).astype(np.int32)
    Tmax = 128
    r = oracle.tree_merge_chains(ct, cq, cl, Tmax)
    dev = cuda_device
    tsd.device_status(dev).zero_()
    t = tsd.tree_merge_chains(*(torch.from_numpy(a).to(dev) for a in (ct, cq, cl)), Tmax=Tmax)
    flagged = (r["status"] != 0).any()
    assert bool(_status(dev) & tsd.binding.DEV_BAD_TREE) == bool(flagged)
    tsd.device_status(dev).zero_()
    assert (t.n_nodes.cpu().numpy() == r["n_nodes"]).all()
    for b in range(B):
        T = int(r["n_nodes"][b])
        if T < 0:
            continue
        assert (t.parent[b, :T].cpu().numpy() == r["parent"][b, :T]).all()
        assert (t.tokens[b, :T].cpu().numpy() == r["tokens"][b, :T]).all()
        assert (t.q_row[b, :T].cpu().numpy() == r["q_row"][b, :T]).all()


def test_merge_overflow(cuda_device):
    dev = cuda_device
    ct = torch.arange(2 * 3 * 5, dtype=torch.int32, device=dev).view(2, 3, 5)   # no sharing
    cq = torch.zeros_like(ct)
    cl = torch.full((2, 3), 5, dtype=torch.int32, device=dev)
    tsd.device_status(dev).zero_()
    t = tsd.tree_merge_chains(ct, cq, cl, Tmax=14)            # 15 nodes needed
    assert _status(dev) & tsd.binding.DEV_BAD_TREE
    assert (t.n_nodes == -1).all().item()
    tsd.device_status(dev).zero_()
