"""GPU parity of tree attention over a paged KV cache (tsd_tree_attention_paged).

The pools are built from the contiguous cache with a random page permutation
(test_oracle_paged._paginate); the oracle's paged attention is the reference,
and the paged call must also reproduce the contiguous call's output exactly
(the kernels see the same keys in the same order).
"""

import numpy as np
import pytest
import torch

import oracle
import tree_speculative_decoding_ancestor_b200 as tsd
from test_oracle_paged import _paginate
from workloads import gen

pytestmark = pytest.mark.gpu


def _status(dev):
    torch.cuda.synchronize(dev)
    return int(tsd.device_status(dev).item())


def _pools(w, page_size, seed):
    kp, table = _paginate(w.k_cache, page_size, np.random.default_rng(seed))
    vp, _ = _paginate(w.v_cache, page_size, np.random.default_rng(seed))
    return kp, vp, table


CASES = [
    # (seed, B, Tmax, Hq, Hkv, D, dtype, page_size)  kernel used
    (41, 3, 40, 32, 4, 128, "bf16", 16),     # tcgen05 128-key rows kernel (320 packed rows)
    (42, 3, 40, 32, 4, 128, "bf16", 128),
    (43, 2, 24, 8, 8, 128, "bf16", 64),      # tcgen05 64-key rows kernel (24 rows)
    (44, 2, 24, 8, 8, 128, "bf16", 256),
    (45, 3, 20, 4, 2, 64, "f32", 32),        # CUDA-core kernel
    (46, 3, 20, 8, 2, 64, "bf16", 16),
]


@pytest.mark.parametrize("case", CASES, ids=[f"s{c[0]}_p{c[7]}" for c in CASES])
def test_paged_attention_parity(cuda_device, case):
    seed, B, Tmax, Hq, Hkv, D, dtype, ps = case
    w = gen.random_workload(seed, B=B, Tmax=Tmax, Hq=Hq, Hkv=Hkv, D=D, P_max=700, V=8,
                            dtype=dtype, min_nodes=1)
    kp, vp, table = _pools(w, ps, seed)
    dev = cuda_device
    d = {k: getattr(w, k).to(dev) for k in ("parent", "n_nodes", "prefix_len", "q", "k_cache",
                                            "v_cache")}
    tree = tsd.tree_mask_build(d["parent"], d["n_nodes"])
    tsd.device_status(dev).zero_()
    got = tsd.tree_attention_paged(d["q"], kp.to(dev), vp.to(dev), table.to(dev),
                                   d["prefix_len"], d["n_nodes"], tree.mask)
    flat = tsd.tree_attention(d["q"], d["k_cache"], d["v_cache"], d["prefix_len"], d["n_nodes"],
                              tree.mask)
    assert _status(dev) == 0
    ref = oracle.tree_attention_paged(w.q, kp, vp, table, ps, w.prefix_len, w.n_nodes, w.parent,
                                      w.scale)
    tol = 1e-4 if dtype == "f32" else 2e-2
    g = got.float().cpu().numpy()
    f = flat.float().cpu().numpy()
    for b in range(B):
        T = int(w.n_nodes[b])
        assert np.abs(g[b, :T] - ref[b, :T]).max() <= tol
        assert np.array_equal(g[b, :T], f[b, :T])


@pytest.mark.parametrize("case", CASES[:2], ids=[f"s{c[0]}_p{c[7]}" for c in CASES[:2]])
def test_paged_attention_parity_paired_rows_kernel(cuda_device, case, monkeypatch):
    # the 64-key rows kernel (two CTAs per SM) instead of the default 128-key one
    monkeypatch.setenv("TSD_ATTN_ROWS_VARIANT", "2")
    test_paged_attention_parity(cuda_device, case)


@pytest.mark.parametrize("case", CASES[2:4], ids=[f"s{c[0]}_p{c[7]}" for c in CASES[2:4]])
def test_paged_attention_parity_small_on_keysplit_kernel(cuda_device, case, monkeypatch):
    monkeypatch.setenv("TSD_ATTN_SMALL_VARIANT", "keysplit")
    test_paged_attention_parity(cuda_device, case)


@pytest.mark.parametrize("D,dtype", [(128, "bf16"), (64, "f32")])
def test_bad_page_is_flagged(cuda_device, D, dtype):
    w = gen.random_workload(47, B=2, Tmax=24, Hq=16, Hkv=2, D=D, P_max=300, V=8, dtype=dtype,
                            ragged=False, P_min=200)
    kp, vp, table = _pools(w, 64, 47)
    table[1, 1] = kp.shape[0] + 5            # a prefix page of sequence 1 out of range
    dev = cuda_device
    d = {k: getattr(w, k).to(dev) for k in ("parent", "n_nodes", "prefix_len", "q")}
    tree = tsd.tree_mask_build(d["parent"], d["n_nodes"])
    tsd.device_status(dev).zero_()
    tsd.tree_attention_paged(d["q"], kp.to(dev), vp.to(dev), table.to(dev), d["prefix_len"],
                             d["n_nodes"], tree.mask)
    assert _status(dev) & tsd.binding.DEV_BAD_PAGE
    tsd.device_status(dev).zero_()


def test_host_checks(cuda_device):
    lib = tsd.load_library()
    z = torch.zeros(64, dtype=torch.int32, device=cuda_device)
    p = z.data_ptr()
    s = torch.cuda.current_stream().cuda_stream
    # page size not a power of two, and below 16
    for ps in (48, 8):
        assert lib.tsd_tree_attention_paged(p, p, p, p, 4, ps, 2, p, p, p, 1, 4, 2, 2, 64, 0.1, 1,
                                            p, None, 0, None, s) == -2
    # no block table
    assert lib.tsd_tree_attention_paged(p, p, p, None, 4, 16, 2, p, p, p, 1, 4, 2, 2, 64, 0.1, 1,
                                        p, None, 0, None, s) == -1


def test_full_size_paged_gqa70b(cuda_device):
    w = gen.config_workload(3)
    kp, vp, table = _pools(w, 128, 3)
    dev = cuda_device
    d = {k: getattr(w, k).to(dev) for k in ("parent", "n_nodes", "prefix_len", "q")}
    tree = tsd.tree_mask_build(d["parent"], d["n_nodes"])
    out = tsd.tree_attention_paged(d["q"], kp.to(dev), vp.to(dev), table.to(dev),
                                   d["prefix_len"], d["n_nodes"], tree.mask)
    assert _status(dev) == 0
    rng = np.random.default_rng(3)
    rows = [(int(rng.integers(w.B)), 0, int(rng.integers(w.Hq))) for _ in range(24)]
    rows = [(b, int(rng.integers(int(w.n_nodes[b]))), h) for b, _, h in rows]
    ref = oracle.tree_attention_rows(w.q, w.k_cache, w.v_cache, w.prefix_len, w.n_nodes,
                                     w.parent, w.scale, rows)
    got = out.float().cpu().numpy()
    err = max(float(np.abs(got[b, u, h] - ref[i]).max()) for i, (b, u, h) in enumerate(rows))
    assert err <= 2e-2, err
