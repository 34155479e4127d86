"""Host-side parts of bench.py that need no GPU: the parity record (the GPU
step's outputs against the oracle's) and the step roofline's byte count.
The "GPU outputs" here are the oracle's own results in the shapes the step
holds, so the record must read exact; planted differences must show."""

import types

import numpy as np
import pytest
import torch

import bench
import oracle
from workloads import gen


def _fake_step(w):
    att = torch.from_numpy(oracle.workload_attention(w)).to(
        torch.bfloat16 if w.dtype == "bf16" else torch.float32)
    res = {}
    for mode, fn in (("greedy", oracle.workload_greedy), ("stochastic", oracle.workload_stochastic)):
        r = fn(w)
        res[mode] = types.SimpleNamespace(
            n_accepted=torch.from_numpy(r["n_accepted"].astype(np.int32)),
            out_path=torch.from_numpy(r["out_path"].astype(np.int32)),
            out_tokens=torch.from_numpy(r["out_tokens"].astype(np.int32)))
    return types.SimpleNamespace(out=att, g=res["greedy"], s=res["stochastic"])


@pytest.fixture(scope="module")
def case():
    w = gen.random_workload(5, B=4, Tmax=12, Hq=4, Hkv=2, D=64, P_max=80, dtype="f32", V=16,
                            min_nodes=0)
    ref = []
    bench.cpu_baseline(w, budget_s=1e9, keep=ref)
    return w, ref


def test_parity_record_exact_on_oracle_outputs(case):
    w, ref = case
    rec = bench.parity_record(w, _fake_step(w), ref)
    assert rec["sequences"] == w.B
    assert rec["attn_rows_compared"] == int(w.n_nodes.sum()) * w.Hq
    assert rec["attn_max_abs"] < 1e-6 and rec["ok"]
    assert rec["greedy"]["mismatches"] == 0 and rec["stochastic"]["mismatches"] == 0


def test_parity_record_sees_planted_differences(case):
    w, ref = case
    b = int(np.argmax(w.n_nodes.numpy()))
    st = _fake_step(w)
    st.out[b, 0, 1, 3] += 0.01
    st.g.out_tokens[b, 0] += 1
    k = int(st.s.n_accepted[b])
    st.s.out_tokens[b, k] += 1
    rec = bench.parity_record(w, st, ref)
    assert not rec["attn_ok"] and abs(rec["attn_max_abs"] - 0.01) < 1e-3
    assert rec["greedy"]["mismatches"] == 1
    assert rec["stochastic"]["mismatches"] + rec["stochastic"]["excused"] == 1
    assert not rec["ok"]


def test_verify_traffic_counts_rows_on_the_path():
    # one sequence: root -> 0 -> 1 (a chain) plus a second root child 2
    w = gen.random_workload(6, B=1, Tmax=3, V=8, min_nodes=3, ragged=False,
                            with_attention=False)
    w.parent[0] = torch.tensor([-1, 0, -1], dtype=torch.int32)
    w.q_row[0] = torch.tensor([0, 1, 0], dtype=torch.int32)
    row = w.V * 4
    res = lambda n, path: types.SimpleNamespace(  # noqa: E731
        n_accepted=torch.tensor([n], dtype=torch.int32),
        out_path=torch.tensor([path + [-1] * (3 - len(path))], dtype=torch.int32))
    # greedy: the rows of the root and of every fully matched node.  Node 0
    # matches the root row's argmax, node 1 node 0's, node 2 does not: the
    # root's, node 0's and node 1's rows (node 1's argmax is the bonus token)
    w.tokens[0] = torch.tensor([3, 5, 1], dtype=torch.int32)
    w.logits[0].zero_()
    w.logits[0, 0, 3] = 1.0
    w.logits[0, 1, 5] = 1.0
    w.logits[0, 2, 7] = 1.0
    st = types.SimpleNamespace(g=res(2, [0, 1]), s=res(0, []))
    vb = bench.verify_traffic(w, st)
    assert vb["greedy"] == 3 * row
    w.tokens[0, 0] = 4   # nothing matches: the root's row alone
    assert bench.verify_traffic(w, st)["greedy"] == 1 * row
    w.tokens[0, 0] = 3
    # stochastic, nothing accepted: root row + the root children's q row (shared)
    assert vb["stochastic"] == 2 * row
    # stochastic, node 0 then node 1 accepted: root row + q row 0; node 0's row +
    # q row 1; node 1's row (a leaf: no children tried)
    st = types.SimpleNamespace(g=res(0, []), s=res(2, [0, 1]))
    assert bench.verify_traffic(w, st)["stochastic"] == 5 * row


def test_input_copies_defeat_the_l2():
    # each workload's inputs are rotated over enough device copies that the
    # copies read since a copy's last use exceed twice the L2; the tiny one
    # cannot be, and falls back to the flush
    for name in ("llama7b", "merge", "gqa70b", "long32k"):
        w = gen.config_workload(gen.WORKLOAD_NAMES[name])
        n = bench.input_sets_for(w)
        nb = bench.input_bytes(w)
        assert n >= 2 and (n - 1) * nb >= 2 * bench.L2_BYTES, (name, n, nb)
        assert n * nb <= 4e9
    assert bench.input_sets_for(gen.config_workload(0)) == 1
