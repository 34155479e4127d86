"""GPU parity of the accepted-path commit (tsd_kv_commit) against the oracle.

The paths come from the oracle's verifiers (never from the CUDA path); both
sides move the same rows and must agree byte for byte.
"""

import numpy as np
import pytest
import torch

import oracle
import tree_speculative_decoding_ancestor_b200 as tsd
from workloads import gen

pytestmark = pytest.mark.gpu


def _raw(t):
    t = t.detach().cpu().contiguous()
    return t.view(torch.int16).numpy() if t.dtype == torch.bfloat16 else t.numpy()


def _oracle_paths(w, mode):
    r = oracle.workload_greedy(w) if mode == "greedy" else oracle.workload_stochastic(w)
    return r["out_path"].astype(np.int32), r["n_accepted"].astype(np.int32)


def _run(w, path, nacc, dev):
    k, v = w.k_cache.to(dev), w.v_cache.to(dev)
    res = tsd.VerifyResult(torch.zeros((w.B, w.Tmax + 1), dtype=torch.int32, device=dev),
                           torch.from_numpy(path).to(dev), torch.from_numpy(nacc).to(dev))
    newp = tsd.kv_commit(k, v, w.prefix_len.to(dev), res)
    torch.cuda.synchronize(dev)
    return k, v, newp


@pytest.mark.parametrize("seed,dtype,D,mode", [(21, "bf16", 64, "greedy"),
                                               (22, "bf16", 128, "stochastic"),
                                               (23, "f32", 64, "stochastic"),
                                               (24, "bf16", 128, "greedy")])
def test_commit_matches_oracle(cuda_device, seed, dtype, D, mode):
    w = gen.random_workload(seed, B=12, Tmax=40, Hq=4, Hkv=2, D=D, P_max=300, V=12,
                            dtype=dtype, min_nodes=0, max_children=2, max_depth=12,
                            token_mode="topk", q_sigma=0.1)
    path, nacc = _oracle_paths(w, mode)
    assert (nacc > 0).any()
    want = oracle.kv_commit(w.k_cache, w.v_cache, w.prefix_len, path, nacc)
    tsd.device_status(cuda_device).zero_()
    k, v, newp = _run(w, path, nacc, cuda_device)
    assert (_raw(k) == want["k_cache"].view(_raw(k).dtype)).all()
    assert (_raw(v) == want["v_cache"].view(_raw(v).dtype)).all()
    assert (newp.cpu().numpy() == want["new_prefix"]).all()
    assert int(tsd.device_status(cuda_device).item()) == 0


@pytest.mark.parametrize("dtype,D", [("bf16", 128), ("f32", 128)])
def test_deep_chain_uses_large_staging(cuda_device, dtype, D):
    # Tmax = 128 chain, every other node accepted from the deep end: the
    # staging buffer is 2 x 128 rows (64 KB bf16, 128 KB fp32).
    w = gen.random_workload(25, B=2, Tmax=128, Hq=2, Hkv=1, D=D, P_max=50, V=8, dtype=dtype,
                            ragged=False, max_children=1, max_depth=128)
    path = np.full((2, 128), -7, dtype=np.int32)
    path[0, :64] = np.arange(1, 128, 2)
    path[1, :128] = np.arange(128)
    nacc = np.array([64, 128], dtype=np.int32)
    want = oracle.kv_commit(w.k_cache, w.v_cache, w.prefix_len, path, nacc)
    k, v, newp = _run(w, path, nacc, cuda_device)
    assert (_raw(k) == want["k_cache"].view(_raw(k).dtype)).all()
    assert (_raw(v) == want["v_cache"].view(_raw(v).dtype)).all()
    assert (newp.cpu().numpy() == want["new_prefix"]).all()


def test_skipped_and_malformed_sequences(cuda_device):
    w = gen.random_workload(26, B=4, Tmax=8, Hq=2, Hkv=2, D=64, P_max=20, V=8, ragged=False)
    path = np.tile(np.array([[0, 2, 3, 0, 0, 0, 0, 0]], dtype=np.int32), (4, 1))
    path[2, :3] = [3, 2, 5]                    # not increasing
    nacc = np.array([3, -1, 3, 0], dtype=np.int32)
    want = oracle.kv_commit(w.k_cache, w.v_cache, w.prefix_len, path, nacc)
    assert list(want["status"]) == [0, 0, oracle.BAD_PATH, 0]
    tsd.device_status(cuda_device).zero_()
    k, v, newp = _run(w, path, nacc, cuda_device)
    assert (_raw(k) == want["k_cache"].view(_raw(k).dtype)).all()
    assert (_raw(v) == want["v_cache"].view(_raw(v).dtype)).all()
    assert (newp.cpu().numpy() == want["new_prefix"]).all()
    assert int(tsd.device_status(cuda_device).item()) == tsd.binding.DEV_BAD_PATH


def test_host_errors(cuda_device):
    lib = tsd.load_library()
    k = torch.zeros((1, 1, 8, 6), dtype=torch.bfloat16, device=cuda_device)
    i32 = torch.zeros(8, dtype=torch.int32, device=cuda_device)
    p = lambda t: t.data_ptr()  # noqa: E731
    s = torch.cuda.current_stream().cuda_stream
    args = (p(k), p(k), p(i32), p(i32), p(i32), 1, 8, 1)
    assert lib.tsd_kv_commit(*args, 6, 8, 1, p(i32), None, s) == -2      # 12-byte rows
    assert lib.tsd_kv_commit(*args, 8, 8, 7, p(i32), None, s) == -3      # dtype
    assert lib.tsd_kv_commit(*args, 8, 8, 1, None, None, s) == -1        # no output
    kk = torch.zeros(64 + 8, dtype=torch.bfloat16, device=cuda_device)
    assert lib.tsd_kv_commit(kk.data_ptr() + 2, p(k), p(i32), p(i32), p(i32), 1, 8, 1, 8, 4, 1,
                             p(i32), None, s) == -6                        # misaligned


@pytest.mark.parametrize("cfg", [3, 4])
def test_full_size_commit(cuda_device, cfg):
    w = gen.config_workload(cfg)
    mode = "stochastic" if "stochastic" in w.verify else "greedy"
    path, nacc = _oracle_paths(w, mode)
    k, v, newp = _run(w, path, nacc, cuda_device)
    want = oracle.kv_commit(w.k_cache, w.v_cache, w.prefix_len, path, nacc)
    assert (newp.cpu().numpy() == want["new_prefix"]).all()
    kg, vg = _raw(k), _raw(v)
    kw = want["k_cache"].view(kg.dtype)
    vw = want["v_cache"].view(vg.dtype)
    k0 = _raw(w.k_cache)
    for b in range(w.B):
        P, T = int(w.prefix_len[b]), int(w.n_nodes[b])
        # the committed rows and the rest of the tree region, all heads
        assert (kg[b, :, P:P + T] == kw[b, :, P:P + T]).all()
        assert (vg[b, :, P:P + T] == vw[b, :, P:P + T]).all()
        # a sample of prefix rows is untouched
        assert (kg[b, :, :P:97] == k0[b, :, :P:97]).all()
