"""Pins of the oracle's paged-KV attention (CPU only).

A paged cache (SpecInfer explainer, "実運用への応用" / "vLLMとの関連": tree
verification combined with PagedAttention's block-wise KV memory) holds the
same logical cache in fixed-size physical pages named by a block table.  The
pin: the test builds the pool from a contiguous cache with torch indexing and
a random page permutation, and the oracle's paged attention must equal its
contiguous attention -- already pinned against the definition -- bit for bit.
"""

import numpy as np
import pytest
import torch

import oracle
from workloads import gen


def _paginate(cache, page_size, rng, spare=3):
    """[B][Hkv][Lmax][D] -> pool [num_pages][Hkv][page_size][D], block table,
    with the physical pages shuffled and a few unused pages in the pool."""
    B, Hkv, Lmax, D = cache.shape
    nblk = (Lmax + page_size - 1) // page_size
    padded = torch.zeros((B, Hkv, nblk * page_size, D), dtype=cache.dtype)
    padded[:, :, :Lmax] = cache
    blocks = padded.view(B, Hkv, nblk, page_size, D).permute(0, 2, 1, 3, 4)  # [B][nblk][Hkv][ps][D]
    logical = blocks.reshape(B * nblk, Hkv, page_size, D)
    n_pages = B * nblk + spare
    perm = torch.from_numpy(rng.permutation(n_pages)[:B * nblk])
    pool = torch.randn((n_pages, Hkv, page_size, D)).to(cache.dtype)
    pool[perm] = logical
    table = perm.view(B, nblk).to(torch.int32)
    return pool, table


@pytest.mark.parametrize("seed,dtype,page_size", [(31, "bf16", 16), (32, "f32", 64),
                                                  (33, "bf16", 128), (34, "bf16", 256)])
def test_paged_equals_contiguous(seed, dtype, page_size):
    w = gen.random_workload(seed, B=3, Tmax=20, Hq=4, Hkv=2, D=32, P_max=300, V=8,
                            dtype=dtype, min_nodes=0)
    rng = np.random.default_rng(seed)
    kp, table = _paginate(w.k_cache, page_size, rng)
    vp, _ = _paginate(w.v_cache, page_size, np.random.default_rng(seed))
    want = oracle.workload_attention(w)
    got = oracle.tree_attention_paged(w.q, kp, vp, table, page_size, w.prefix_len, w.n_nodes,
                                      w.parent, w.scale)
    Lmax = w.k_cache.shape[2]
    assert got.shape == want.shape
    for b in range(w.B):
        T = int(w.n_nodes[b])
        assert np.array_equal(got[b, :T], want[b, :T])
    # the gathered cache itself, up to the contiguous length
    k, v = oracle.gather_pages(kp, vp, table, page_size, table.shape[1] * page_size)
    assert np.array_equal(k[:, :, :Lmax], oracle._np(w.k_cache))
    assert np.array_equal(v[:, :, :Lmax], oracle._np(w.v_cache))


def test_a_swapped_page_changes_the_result():
    w = gen.random_workload(35, B=1, Tmax=8, Hq=2, Hkv=1, D=16, P_max=60, V=8, dtype="f32",
                            ragged=False, P_min=60)
    kp, table = _paginate(w.k_cache, 16, np.random.default_rng(0))
    vp, _ = _paginate(w.v_cache, 16, np.random.default_rng(0))
    ref = oracle.tree_attention_paged(w.q, kp, vp, table, 16, w.prefix_len, w.n_nodes, w.parent,
                                      w.scale)
    bad = table.clone()
    bad[0, [0, 1]] = bad[0, [1, 0]]
    got = oracle.tree_attention_paged(w.q, kp, vp, bad, 16, w.prefix_len, w.n_nodes, w.parent,
                                      w.scale)
    # swapping two prefix pages permutes keys with their values: the prefix
    # is a set, so the result is unchanged ...
    np.testing.assert_allclose(got, ref, rtol=0, atol=1e-12)
    # ... but swapping a prefix page with the page holding the tree is not
    last = (int(w.prefix_len[0])) // 16
    bad = table.clone()
    bad[0, [0, last]] = bad[0, [last, 0]]
    got = oracle.tree_attention_paged(w.q, kp, vp, bad, 16, w.prefix_len, w.n_nodes, w.parent,
                                      w.scale)
    assert not np.allclose(got, ref)
