"""GPU parity of the CUDA path against the CPU oracle, called through the C
ABI (the ctypes binding of libtsd.so).

* mask: bit-exact on random ragged trees (Tmax up to 128) and malformed ones;
* attention: max-abs 2e-2 (bf16) / 1e-4 (fp32) against the fp64 oracle on
  small and ragged shapes that span several key tiles and a ragged tail,
  with poisoned padding, and on sampled rows at the five workload sizes;
* greedy verify: bit-exact tokens and paths;
* stochastic verify: bit-exact except boundary-flagged draws (< 1e-4).
"""

import numpy as np
import pytest
import torch

import oracle
import tree_speculative_decoding_ancestor_b200 as tsd
from workloads import gen

from gpu_util import (check_attention, check_greedy, check_mask, check_stochastic, poison,
                      run_tree, to_dev)

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True)
def _clear_status(cuda_device):
    tsd.device_status(cuda_device).zero_()
    yield


def _status(dev):
    torch.cuda.synchronize(dev)
    return int(tsd.device_status(dev).item())


# ------------------------------------------------------------------ mask
@pytest.mark.parametrize("Tmax", [1, 6, 31, 32, 33, 64, 100, 128])
def test_mask_random_trees(cuda_device, Tmax):
    w = gen.random_workload(Tmax, B=9, Tmax=Tmax, min_nodes=0, max_children=5,
                            max_depth=Tmax, with_attention=False, V=8)
    d = to_dev(w, cuda_device)
    tree = run_tree(d)
    check_mask(w, tree)
    assert _status(cuda_device) == 0


def test_mask_malformed(cuda_device):
    parent = torch.tensor([[-1, 0, 1, -1], [0, -1, -1, -1], [-1, 3, -1, -1], [-1, -1, 0, 7]],
                          dtype=torch.int32)
    n_nodes = torch.tensor([4, 1, 3, 4], dtype=torch.int32)
    tree = tsd.tree_mask_build(parent.to(cuda_device), n_nodes.to(cuda_device))
    fc = tree.first_child.cpu()
    assert fc[0, 0] == 0 and (fc[1:, 0] == -2).all()
    assert (tree.mask.cpu()[1:] == 0).all()
    assert _status(cuda_device) & 1
    # n_nodes out of range
    tsd.device_status(cuda_device).zero_()
    tree = tsd.tree_mask_build(parent.to(cuda_device),
                               torch.tensor([5, -1, 0, 0], dtype=torch.int32).to(cuda_device))
    assert (tree.first_child.cpu()[:2, 0] == -2).all()
    assert _status(cuda_device) & 1


# ------------------------------------------------------------- attention
ATTN_CASES = [
    # (seed, B, Tmax, Hq, Hkv, D, P_max, dtype)
    (1, 3, 6, 4, 4, 64, 64, "f32"),
    (2, 2, 20, 8, 8, 128, 300, "bf16"),
    (3, 4, 24, 16, 2, 128, 513, "bf16"),
    (4, 2, 64, 16, 2, 128, 700, "bf16"),
    (5, 3, 17, 12, 3, 64, 129, "bf16"),
    (6, 2, 128, 8, 1, 128, 260, "bf16"),
    (7, 3, 33, 6, 2, 64, 97, "f32"),
    (8, 2, 128, 32, 8, 128, 1100, "bf16"),
]


@pytest.mark.parametrize("case", ATTN_CASES, ids=[f"s{c[0]}" for c in ATTN_CASES])
def test_attention_parity(cuda_device, case):
    seed, B, Tmax, Hq, Hkv, D, P_max, dtype = case
    w = gen.random_workload(seed, B=B, Tmax=Tmax, Hq=Hq, Hkv=Hkv, D=D, P_max=P_max, dtype=dtype,
                            min_nodes=1, max_children=4, max_depth=12, lmax_pad=37, V=16)
    d = to_dev(w, cuda_device)
    poison(w, d)
    tree = run_tree(d)
    sentinel = 1234.0
    out = torch.full_like(d["q"], sentinel)
    tsd.tree_attention(d["q"], d["k_cache"], d["v_cache"], d["prefix_len"], d["n_nodes"],
                       tree.mask, out=out)
    check_attention(w, out, sentinel=sentinel)
    assert _status(cuda_device) == 0


# cases with more than 128 packed rows, on the 64-key rows kernel (two CTAs
# per SM) instead of the default 128-key one (one CTA per SM)
ROWS_CASES = [c for c in ATTN_CASES if c[7] == "bf16" and c[5] == 128 and c[2] * c[3] // c[4] > 128]


@pytest.mark.parametrize("case", ROWS_CASES, ids=[f"s{c[0]}" for c in ROWS_CASES])
def test_attention_parity_paired_rows_kernel(cuda_device, case, monkeypatch):
    monkeypatch.setenv("TSD_ATTN_ROWS_VARIANT", "2")
    test_attention_parity(cuda_device, case)


@pytest.mark.parametrize("case", ROWS_CASES, ids=[f"s{c[0]}" for c in ROWS_CASES])
def test_attention_parity_rows_kernel_paired_softmax(cuda_device, case, monkeypatch):
    # more than 128 packed rows on the 128-key rows kernel with two softmax
    # warps per TMEM lane quarter
    monkeypatch.setenv("TSD_ATTN_SOFTMAX_WARPS", "2")
    test_attention_parity(cuda_device, case)


SMALL_CASES = [c for c in ATTN_CASES if c[7] == "bf16" and c[5] == 128 and c[2] * c[3] // c[4] <= 128]


@pytest.mark.parametrize("case", SMALL_CASES, ids=[f"s{c[0]}" for c in SMALL_CASES])
def test_attention_parity_small_on_keysplit_kernel(cuda_device, case, monkeypatch):
    # at most 128 packed rows, on the key-split kernel instead of the 64-key rows one
    monkeypatch.setenv("TSD_ATTN_SMALL_VARIANT", "keysplit")
    test_attention_parity(cuda_device, case)


# Full trees at the row-block boundary: 32 nodes x G = 4 is exactly 128
# packed rows, the largest query block of the small-shape kernels; 33 nodes
# give 132 rows, the 128-key rows kernel with a second block of 4 real rows.
@pytest.mark.parametrize("Tmax,env", [(32, None), (32, ("TSD_ATTN_SMALL_VARIANT", "keysplit")),
                                      (33, None), (33, ("TSD_ATTN_ROWS_VARIANT", "2"))],
                         ids=["128-rows", "128-rows-keysplit", "132-rows", "132-rows-paired"])
def test_attention_parity_at_the_row_block_boundary(cuda_device, Tmax, env, monkeypatch):
    if env:
        monkeypatch.setenv(*env)
    w = gen.random_workload(90 + Tmax, B=2, Tmax=Tmax, Hq=8, Hkv=2, D=128, P_max=400,
                            dtype="bf16", min_nodes=Tmax, max_children=4, max_depth=12,
                            lmax_pad=37, V=16)
    assert (w.n_nodes == Tmax).all()
    d = to_dev(w, cuda_device)
    poison(w, d)
    tree = run_tree(d)
    sentinel = 1234.0
    out = torch.full_like(d["q"], sentinel)
    tsd.tree_attention(d["q"], d["k_cache"], d["v_cache"], d["prefix_len"], d["n_nodes"],
                       tree.mask, out=out)
    check_attention(w, out, sentinel=sentinel)
    assert _status(cuda_device) == 0


# Forced key-range split counts (TSD_ATTN_SPLITS) on every kernel: one split
# takes each kernel's direct normalised write, one key tile per split the
# partials + log-sum-exp combine (and leaves the key-split kernel's second
# softmax group without tiles).  The large shape has up to 256 packed rows
# per (sequence, KV head) -- two row blocks on the 128-key rows kernel, the
# plan the 70B-GQA benchmark runs with one split -- and is compared on every
# row.
LARGE = dict(seed=81, B=4, Tmax=64, Hq=32, Hkv=8, D=128, P_max=1500, P_min=900, min_nodes=36)
SMALL = dict(seed=82, B=3, Tmax=24, Hq=16, Hkv=4, D=128, P_max=900, P_min=300, min_nodes=8)
FORCED = [
    # (shape, environment, expected kernel)
    ("large", {}, "rows128"),
    ("large", {"TSD_ATTN_ROWS_VARIANT": "2"}, "rows64"),
    ("large", {"TSD_ATTN_SOFTMAX_WARPS": "2"}, "rows128x2"),
    ("small", {}, "rows64"),
    ("small", {"TSD_ATTN_SMALL_VARIANT": "keysplit"}, "keysplit"),
    ("small", {"TSD_FORCE_PATH": "simt"}, "simt"),
]


def _shape_workload(name):
    c = dict(LARGE if name == "large" else SMALL)
    return gen.random_workload(c.pop("seed"), dtype="bf16", max_children=4, max_depth=12,
                               lmax_pad=37, V=16, **c)


FORCED_IDS = [f"{f[0]}-{f[2]}" for f in FORCED]


@pytest.mark.parametrize("splits", ["1", "3", "64"])
@pytest.mark.parametrize("forced", FORCED, ids=FORCED_IDS)
def test_attention_parity_forced_splits(cuda_device, forced, splits, monkeypatch):
    shape, env, kernel = forced
    for k, v in env.items():
        monkeypatch.setenv(k, v)
    monkeypatch.setenv("TSD_ATTN_SPLITS", splits)
    w = _shape_workload(shape)
    sms = torch.cuda.get_device_properties(cuda_device).multi_processor_count
    plan = tsd.attention_plan(w.B, w.Tmax, w.Hq, w.Hkv, w.D, w.Lmax, torch.bfloat16, sms)
    assert plan["kernel"] == kernel
    tiles = -(-w.Lmax // (128 if kernel in ("rows128", "rows128x2", "keysplit") else
                          64 if kernel == "rows64" else 32))
    assert plan["splits"] == min(int(splits), tiles if kernel != "simt" else plan["splits"])
    if shape == "large" and kernel in ("rows128", "rows128x2"):
        assert plan["row_blocks"] == 2 and max(w.n_nodes.tolist()) * w.G > 128
    d = to_dev(w, cuda_device)
    poison(w, d)
    tree = run_tree(d)
    out = torch.full_like(d["q"], 1234.0)
    tsd.tree_attention(d["q"], d["k_cache"], d["v_cache"], d["prefix_len"], d["n_nodes"],
                       tree.mask, out=out)
    check_attention(w, out, sentinel=1234.0)
    assert _status(cuda_device) == 0


@pytest.mark.parametrize("splits", ["1", "2"])
@pytest.mark.parametrize("forced", FORCED, ids=FORCED_IDS)
def test_attention_row_without_keys_is_zero(cuda_device, forced, splits, monkeypatch):
    # A caller-supplied mask row without the node's own bit, in a sequence with
    # no prefix, leaves that query row no key at all: every kernel writes it as
    # zeros, whatever the split count; the other rows keep the oracle's values.
    shape, env, kernel = forced
    for k, v in env.items():
        monkeypatch.setenv(k, v)
    monkeypatch.setenv("TSD_ATTN_SPLITS", splits)
    w = _shape_workload(shape)
    w.prefix_len[0] = 0
    ref = oracle.workload_attention(w)
    d = to_dev(w, cuda_device)
    tree = run_tree(d)
    u0 = 0   # the root's first child: its only key is itself
    tree.mask[0, u0].zero_()
    out = tsd.tree_attention(d["q"], d["k_cache"], d["v_cache"], d["prefix_len"], d["n_nodes"],
                             tree.mask)
    got = out.float().cpu()
    assert (got[0, u0] == 0).all().item()
    ref[0, u0] = got[0, u0].numpy()
    check_attention(w, out, ref=ref)
    assert _status(cuda_device) == 0


def test_attention_empty_trees_and_prefix(cuda_device):
    # T_b = 0 sequences, P_b = 0 sequences, and a single-node tree with no prefix
    w = gen.random_workload(21, B=4, Tmax=8, Hq=4, Hkv=2, D=128, P_max=50, dtype="bf16",
                            min_nodes=0, V=16)
    w.n_nodes[0] = 0
    w.prefix_len[1] = 0
    w.prefix_len[2] = 0
    w.n_nodes[2] = 1
    w2 = gen.random_workload(21, B=4, Tmax=8, Hq=4, Hkv=2, D=128, P_max=50, dtype="bf16",
                             min_nodes=0, V=16)
    # regenerate caches consistent with the edited sizes: reuse, values are random anyway
    d = to_dev(w, cuda_device)
    tree = run_tree(d)
    out = torch.full_like(d["q"], 7.0)
    tsd.tree_attention(d["q"], d["k_cache"], d["v_cache"], d["prefix_len"], d["n_nodes"],
                       tree.mask, out=out)
    check_attention(w, out, sentinel=7.0)
    # one node, no prefix: the output is that node's value row (rounded to bf16)
    o = out.float().cpu()[2, 0]
    v = w.v_cache.float()[2, :, 0].repeat_interleave(2, dim=0)
    assert torch.equal(o, v)
    del w2


def test_attention_bad_prefix_flagged(cuda_device):
    w = gen.random_workload(22, B=2, Tmax=4, Hq=2, Hkv=2, D=64, P_max=20, dtype="bf16",
                            ragged=False, V=16)
    d = to_dev(w, cuda_device)
    tree = run_tree(d)
    d["prefix_len"][1] = w.Lmax  # P + T > Lmax
    out = torch.full_like(d["q"], 3.0)
    tsd.tree_attention(d["q"], d["k_cache"], d["v_cache"], d["prefix_len"], d["n_nodes"],
                       tree.mask, out=out)
    assert _status(cuda_device) & 8
    assert (out[1].float() == 3.0).all().item()


def test_attention_host_errors(cuda_device):
    lib = tsd.load_library()
    q = torch.zeros(1, 4, 4, 64, dtype=torch.bfloat16, device=cuda_device)
    kv = torch.zeros(1, 4, 8, 64, dtype=torch.bfloat16, device=cuda_device)
    i32 = torch.zeros(4, dtype=torch.int32, device=cuda_device)
    args = [q.data_ptr(), kv.data_ptr(), kv.data_ptr(), i32.data_ptr(), i32.data_ptr(),
            i32.data_ptr()]
    s = torch.cuda.current_stream().cuda_stream
    # Hq % Hkv != 0
    assert lib.tsd_tree_attention(*args, 1, 4, 4, 3, 64, 8, 0.1, 1, q.data_ptr(), None, 0, None,
                                  s) == -2
    # head_dim not supported
    assert lib.tsd_tree_attention(*args, 1, 4, 4, 4, 80, 8, 0.1, 1, q.data_ptr(), None, 0, None,
                                  s) == -3
    # misaligned pointer
    assert lib.tsd_tree_attention(q.data_ptr() + 2, *args[1:], 1, 4, 4, 4, 64, 8, 0.1, 1,
                                  q.data_ptr(), None, 0, None, s) == -6
    # empty batch launches nothing
    assert lib.tsd_tree_attention(*args, 0, 4, 4, 4, 64, 8, 0.1, 1, q.data_ptr(), None, 0, None,
                                  s) == 0


# ----------------------------------------------------------------- verify
VERIFY_CASES = [
    # (seed, B, Tmax, V, token_mode, temperature)
    (31, 16, 6, 32, "sample", 1.0),
    (32, 8, 24, 1000, "sample", 0.7),
    (33, 8, 64, 4099, "topk", 1.0),
    (34, 4, 128, 32000, "sample", 1.0),
    (35, 32, 20, 5, "sample", 1.3),
    (36, 6, 40, 777, "topk", 0.5),
    (37, 2, 16, 128256, "topk", 1.0),    # 32-CTA teams, 4008 entries each
    (38, 3, 12, 50001, "sample", 0.9),   # last chunk ends at V, V % 4 != 0
    (39, 1100, 8, 64, "sample", 1.0),    # more sequences than the grid holds
]


@pytest.mark.parametrize("exchange", ["cluster", "global"])
@pytest.mark.parametrize("case", VERIFY_CASES, ids=[f"s{c[0]}" for c in VERIFY_CASES])
def test_verify_parity(cuda_device, case, exchange, monkeypatch):
    # exchange: the walk's teams as thread-block clusters (the default up to
    # 8 x 4096 vocabulary entries) or as CTAs of a cooperative launch
    seed, B, Tmax, V, mode, temp = case
    if exchange == "global":
        monkeypatch.setenv("TSD_WALK_EXCHANGE", "global")
    elif V > 8 * 4096:
        pytest.skip("the cluster form takes vocabularies up to 32768")
    if seed == 39:   # one-CTA teams that each walk several sequences
        assert tsd.verify_stochastic_plan(B, Tmax, V)["teams"] < B
    w = gen.random_workload(seed, B=B, Tmax=Tmax, V=V, min_nodes=0, max_children=5,
                            max_depth=10, token_mode=mode, q_sigma=0.3, temperature=temp,
                            with_attention=False)
    d = to_dev(w, cuda_device)
    tree = run_tree(d)
    sentinel = -7
    out = tsd.VerifyResult(torch.full((B, Tmax + 1), sentinel, dtype=torch.int32,
                                      device=cuda_device),
                           torch.full((B, Tmax), sentinel, dtype=torch.int32, device=cuda_device),
                           torch.full((B,), sentinel, dtype=torch.int32, device=cuda_device))
    res = tsd.tree_verify_greedy(d["logits"], d["tokens"], d["parent"], d["n_nodes"], tree,
                                 out=out)
    ref = oracle.workload_greedy(w)
    check_greedy(w, res, ref)
    assert (res.out_tokens.cpu().numpy() == ref["out_tokens"]).all()   # untouched = sentinel
    assert (res.out_path.cpu().numpy() == ref["out_path"]).all()
    for t in out:
        t.fill_(sentinel)
    res = tsd.tree_verify_stochastic(d["logits"], temp, d["q_probs"], d["q_row"], d["tokens"],
                                     d["n_nodes"], tree, d["u_accept"], d["u_sample"], out=out)
    ref = oracle.workload_stochastic(w)
    stats = check_stochastic(w, res, ref)
    assert stats["mismatches"] == 0 or stats["excused"] == stats["mismatches"]
    assert _status(cuda_device) == 0


@pytest.mark.parametrize("form", ["walk", "rows"])
@pytest.mark.parametrize("case", VERIFY_CASES + [(40, 6, 48, 700, "match", 1.0)],
                         ids=[f"s{c[0]}" for c in VERIFY_CASES] + ["s40-all-match"])
def test_verify_greedy_forms(cuda_device, case, form, monkeypatch):
    # both greedy forms: the matched-path walk (default) and every row with
    # children + finalize.  "match": every token is its parent row's argmax,
    # so siblings share tokens, whole levels match and the deepest path (ties
    # to the lowest index) decides.
    monkeypatch.setenv("TSD_GREEDY_FORM", form)
    seed, B, Tmax, V, mode, temp = case
    w = gen.random_workload(seed, B=B, Tmax=Tmax, V=V, min_nodes=0, max_children=5,
                            max_depth=10, token_mode="sample" if mode == "match" else mode,
                            q_sigma=0.3, temperature=temp, with_attention=False)
    if mode == "match":
        for b in range(w.B):
            for u in range(int(w.n_nodes[b])):
                w.tokens[b, u] = int(np.argmax(np.asarray(w.logits[b, int(w.parent[b, u]) + 1])))
    d = to_dev(w, cuda_device)
    tree = run_tree(d)
    sentinel = -7
    out = tsd.VerifyResult(torch.full((B, Tmax + 1), sentinel, dtype=torch.int32,
                                      device=cuda_device),
                           torch.full((B, Tmax), sentinel, dtype=torch.int32, device=cuda_device),
                           torch.full((B,), sentinel, dtype=torch.int32, device=cuda_device))
    res = tsd.tree_verify_greedy(d["logits"], d["tokens"], d["parent"], d["n_nodes"], tree,
                                 out=out)
    ref = oracle.workload_greedy(w)
    check_greedy(w, res, ref)
    assert (res.out_tokens.cpu().numpy() == ref["out_tokens"]).all()   # untouched = sentinel
    assert (res.out_path.cpu().numpy() == ref["out_path"]).all()
    if mode == "match":   # the whole deepest path is accepted somewhere
        assert int(res.n_accepted.max()) >= 3
    assert _status(cuda_device) == 0


@pytest.mark.parametrize("exchange", ["cluster", "global"])
def test_verify_many_seeds_stochastic(cuda_device, exchange, monkeypatch):
    # many small trees with accepted paths of every length; counts excusals
    if exchange == "global":
        monkeypatch.setenv("TSD_WALK_EXCHANGE", "global")
    total = dict(mismatches=0, excused=0, decisions=0)
    for seed in range(40, 52):
        w = gen.random_workload(seed, B=64, Tmax=12, V=64, min_nodes=0, max_children=4,
                                max_depth=6, token_mode="sample", q_sigma=0.2,
                                with_attention=False)
        d = to_dev(w, cuda_device)
        tree = run_tree(d)
        res = tsd.tree_verify_stochastic(d["logits"], 1.0, d["q_probs"], d["q_row"], d["tokens"],
                                         d["n_nodes"], tree, d["u_accept"], d["u_sample"])
        s = check_stochastic(w, res)
        for k in total:
            total[k] += s[k]
    assert total["decisions"] > 1000
    assert total["excused"] <= 1e-4 * total["decisions"]


@pytest.mark.parametrize("form", ["walk", "rows"])
def test_verify_malformed_inputs(cuda_device, form, monkeypatch):
    monkeypatch.setenv("TSD_GREEDY_FORM", form)
    w = gen.random_workload(60, B=3, Tmax=6, V=10, min_nodes=3, ragged=False,
                            with_attention=False)
    d = to_dev(w, cuda_device)
    tree = run_tree(d)
    d["tokens"][1, 0] = 10          # token id >= V
    d["q_row"][2, 1] = w.Rq + 3     # q row out of range
    res = tsd.tree_verify_stochastic(d["logits"], 1.0, d["q_probs"], d["q_row"], d["tokens"],
                                     d["n_nodes"], tree, d["u_accept"], d["u_sample"])
    n = res.n_accepted.cpu().tolist()
    assert n[1] == -1 and n[2] == -1 and n[0] >= 0
    assert _status(cuda_device) & (2 | 4) == (2 | 4)
    tsd.device_status(cuda_device).zero_()
    res = tsd.tree_verify_greedy(d["logits"], d["tokens"], d["parent"], d["n_nodes"], tree)
    assert res.n_accepted.cpu().tolist()[1] == -1
    assert _status(cuda_device) & 2
    # malformed tree -> -1 from both verifiers
    d["parent"][0, 2] = 2
    tsd.device_status(cuda_device).zero_()
    tree = run_tree(d)
    res = tsd.tree_verify_greedy(d["logits"], d["tokens"], d["parent"], d["n_nodes"], tree)
    assert res.n_accepted.cpu().tolist()[0] == -1
    assert _status(cuda_device) & 1


# ---------------------------------------------- the five workload sizes
def _sample_rows(w, n, seed):
    rng = np.random.default_rng(seed)
    rows = []
    for _ in range(n):
        b = int(rng.integers(w.B))
        T = int(w.n_nodes[b])
        rows.append((b, int(rng.integers(T)), int(rng.integers(w.Hq))))
    # always include the deepest node of sequence 0 and the last head
    T0 = int(w.n_nodes[0])
    rows.append((0, T0 - 1, w.Hq - 1))
    return rows


@pytest.mark.parametrize("cfg", [3, 4])
def test_config_full_size_paired_softmax(cuda_device, cfg, monkeypatch):
    monkeypatch.setenv("TSD_ATTN_SOFTMAX_WARPS", "2")
    test_config_full_size(cuda_device, cfg)


@pytest.mark.parametrize("cfg", [0, 1, 2, 3, 4])
def test_config_full_size(cuda_device, cfg):
    # The launch the benchmark times (same sizes, same plan), compared with
    # the oracle on every row of the first and last sequence (all nodes, all
    # heads) and on rows sampled from the whole batch.
    w = gen.config_workload(cfg)
    d = to_dev(w, cuda_device)
    tree = run_tree(d)
    check_mask(w, tree)
    out = tsd.tree_attention(d["q"], d["k_cache"], d["v_cache"], d["prefix_len"], d["n_nodes"],
                             tree.mask)
    if cfg == 0:
        check_attention(w, out)
    else:
        rows = _sample_rows(w, 48, cfg)
        for b in sorted({0, w.B - 1}):
            rows += [(b, u, h) for u in range(int(w.n_nodes[b])) for h in range(w.Hq)]
        ref = oracle.tree_attention_rows(w.q, w.k_cache, w.v_cache, w.prefix_len, w.n_nodes,
                                         w.parent, w.scale, rows)
        got = out.float().cpu().numpy()
        err = max(float(np.abs(got[b, u, h] - ref[i]).max()) for i, (b, u, h) in enumerate(rows))
        assert err <= 2e-2, err
        for b in range(w.B):   # rows of padding slots are never written
            assert torch.isfinite(out[b, :int(w.n_nodes[b])].float()).all().item()
    if "greedy" in w.verify:
        check_greedy(w, tsd.tree_verify_greedy(d["logits"], d["tokens"], d["parent"],
                                               d["n_nodes"], tree))
    if "stochastic" in w.verify:
        check_stochastic(w, tsd.tree_verify_stochastic(d["logits"], w.temperature, d["q_probs"],
                                                       d["q_row"], d["tokens"], d["n_nodes"],
                                                       tree, d["u_accept"], d["u_sample"]))
    assert _status(cuda_device) == 0


# ------------------------------------------------- table-driven fp64 exp
def test_table_exp_accuracy(cuda_device, tmp_path):
    """The verifier's bulk fp64 exp (Tang's table-driven method) stays within
    4e-15 relative (a few ulp) of CUDA's exp() on [-60, 0] and at special
    points down to -708, and flushes x < -708 to 0."""
    import os
    import subprocess
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    exe = str(tmp_path / "table_exp_check")
    subprocess.run(["/usr/local/cuda/bin/nvcc", "-O3", "-gencode", "arch=compute_100a,code=sm_100a",
                    "-I", os.path.join(root, "tree_speculative_decoding_ancestor_b200", "csrc"),
                    os.path.join(root, "tests", "cuda", "table_exp_check.cu"), "-o", exe],
                   check=True)
    r = subprocess.run([exe, "4e-15"], capture_output=True, text=True)
    assert r.returncode == 0, r.stdout + r.stderr



def test_verify_greedy_and_stochastic_on_two_streams(cuda_device):
    # The two verify calls read the same inputs and nothing of each other's:
    # run side by side on two streams (each with its own workspace, as the
    # benchmark's step does) they give what they give one after the other.
    w = gen.random_workload(90, B=24, Tmax=48, V=32000, min_nodes=8, max_children=5,
                            max_depth=8, token_mode="sample", q_sigma=1.0,
                            with_attention=False)
    d = to_dev(w, cuda_device)
    tree = run_tree(d)
    B, Tmax = w.B, w.Tmax

    def outs():   # every entry preset, so that the untouched ones compare too
        return tsd.VerifyResult(
            torch.full((B, Tmax + 1), -7, dtype=torch.int32, device=cuda_device),
            torch.full((B, Tmax), -7, dtype=torch.int32, device=cuda_device),
            torch.full((B,), -7, dtype=torch.int32, device=cuda_device))

    g_ref = tsd.tree_verify_greedy(d["logits"], d["tokens"], d["parent"], d["n_nodes"], tree,
                                   out=outs())
    s_ref = tsd.tree_verify_stochastic(d["logits"], w.temperature, d["q_probs"], d["q_row"],
                                       d["tokens"], d["n_nodes"], tree, d["u_accept"],
                                       d["u_sample"], out=outs())
    torch.cuda.synchronize(cuda_device)
    nb = tsd.verify_workspace_size(B, Tmax, w.V)
    ws_g = torch.empty(nb, dtype=torch.uint8, device=cuda_device)
    ws_s = torch.empty(nb, dtype=torch.uint8, device=cuda_device)
    side = torch.cuda.Stream(device=cuda_device)
    main = torch.cuda.current_stream(cuda_device)
    for _ in range(3):
        g_out, s_out = outs(), outs()
        side.wait_stream(main)
        s = tsd.tree_verify_stochastic(d["logits"], w.temperature, d["q_probs"], d["q_row"],
                                       d["tokens"], d["n_nodes"], tree, d["u_accept"],
                                       d["u_sample"], out=s_out, workspace=ws_s)
        with torch.cuda.stream(side):
            g = tsd.tree_verify_greedy(d["logits"], d["tokens"], d["parent"], d["n_nodes"],
                                       tree, out=g_out, workspace=ws_g)
        main.wait_stream(side)
        torch.cuda.synchronize(cuda_device)
        for a, b in ((g, g_ref), (s, s_ref)):
            assert torch.equal(a.n_accepted, b.n_accepted)
            assert torch.equal(a.out_tokens, b.out_tokens)
            assert torch.equal(a.out_path, b.out_path)
    assert _status(cuda_device) == 0
