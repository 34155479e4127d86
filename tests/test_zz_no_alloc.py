"""The allocation-free stochastic verifier (tsd_tree_verify_stochastic_noalloc).

Some callers cannot hand the library a scratch buffer: a serving engine whose
KV-cache pool already owns nearly all device memory, or a caller that reaches
the library through a plain C interface with no device allocator.  This entry
point keeps its scratch in a fixed array inside the library instead.  These
tests call it through the C ABI (ctypes, no Python wrapper in between) and
check that it returns exactly what the workspace entry point returns, and
what the fp64 oracle returns, on two calls in a row (the second call finds
the first call's leftovers in the shared array), and that its fixed scratch
does not limit the shape: a batch with more sequences than the verifier's
grid has teams still runs, one-CTA teams walking several sequences each.

This file is collected last on purpose, so that a run stopping at the first
failure has already run every other test.
"""

import ctypes

import pytest
import torch

import oracle
import tree_speculative_decoding_ancestor_b200 as tsd
from gpu_util import check_stochastic
from workloads import gen

pytestmark = pytest.mark.gpu

TSD_ERR_WORKSPACE = -4


def _inputs(seed, dev, B, Tmax, V):
    w = gen.random_workload(seed, B=B, Tmax=Tmax, V=V, min_nodes=0, max_children=5,
                            max_depth=8, token_mode="sample", q_sigma=0.3,
                            with_attention=False)
    d = {k: getattr(w, k).to(dev) for k in ("parent", "n_nodes", "tokens", "q_row", "logits",
                                            "q_probs", "u_accept", "u_sample")}
    tree = tsd.tree_mask_build(d["parent"], d["n_nodes"])
    return w, d, tree


def _outputs(B, Tmax, dev, fill=-7):
    return tsd.VerifyResult(torch.full((B, Tmax + 1), fill, dtype=torch.int32, device=dev),
                            torch.full((B, Tmax), fill, dtype=torch.int32, device=dev),
                            torch.full((B,), fill, dtype=torch.int32, device=dev))


def _call_noalloc(lib, w, d, tree, out, status, B=None, Tmax=None):
    B = w.B if B is None else B
    Tmax = w.Tmax if Tmax is None else Tmax
    p = lambda t: ctypes.c_void_p(t.data_ptr())  # noqa: E731
    return lib.tsd_tree_verify_stochastic_noalloc(
        p(d["logits"]), w.temperature, p(d["q_probs"]), d["q_probs"].shape[1], p(d["q_row"]),
        p(d["tokens"]), p(d["n_nodes"]), p(tree.first_child), p(tree.next_sibling),
        p(d["u_accept"]), p(d["u_sample"]), B, Tmax, w.V, p(out.out_tokens), p(out.out_path),
        p(out.n_accepted), p(status), torch.cuda.current_stream().cuda_stream)


def test_noalloc_matches_workspace_call_twice(cuda_device):
    lib = tsd.load_library()
    status = torch.zeros(1, dtype=torch.int32, device=cuda_device)
    shapes = [(71, 16, 24, 1000), (72, 9, 64, 32000)]   # two calls in a row
    for seed, B, Tmax, V in shapes:
        w, d, tree = _inputs(seed, cuda_device, B, Tmax, V)
        want = tsd.tree_verify_stochastic(d["logits"], w.temperature, d["q_probs"], d["q_row"],
                                          d["tokens"], d["n_nodes"], tree, d["u_accept"],
                                          d["u_sample"], out=_outputs(B, Tmax, cuda_device))
        got = _outputs(B, Tmax, cuda_device)
        assert _call_noalloc(lib, w, d, tree, got, status) == 0
        torch.cuda.synchronize(cuda_device)
        # identical kernels on identical inputs: exact equality, untouched
        # entries (the -7 fill) included
        assert torch.equal(got.n_accepted, want.n_accepted)
        assert torch.equal(got.out_tokens, want.out_tokens)
        assert torch.equal(got.out_path, want.out_path)
        assert (got.n_accepted >= 0).all().item()
        check_stochastic(w, got, oracle.workload_stochastic(w))
    assert int(status.item()) == 0


def test_noalloc_takes_a_batch_larger_than_the_grid(cuda_device):
    lib = tsd.load_library()
    # 1100 sequences over a 64-token vocabulary: one CTA per team, and more
    # sequences than the teams the device holds at once (the plan caps the
    # teams at that), so teams walk several sequences each and their
    # exchange state runs on from one sequence to the next.
    dev = cuda_device
    B, Tmax, V = 1100, 24, 64
    plan = tsd.verify_stochastic_plan(B, Tmax, V)
    assert plan["ctas_per_team"] == 1
    assert plan["teams"] < B, plan
    w, d, tree = _inputs(77, dev, B=B, Tmax=Tmax, V=V)
    want = tsd.tree_verify_stochastic(d["logits"], w.temperature, d["q_probs"], d["q_row"],
                                      d["tokens"], d["n_nodes"], tree, d["u_accept"],
                                      d["u_sample"], out=_outputs(w.B, w.Tmax, dev))
    status = torch.zeros(1, dtype=torch.int32, device=dev)
    out = _outputs(w.B, w.Tmax, dev)
    torch.cuda.synchronize(dev)
    before = tsd.launch_count()
    assert _call_noalloc(lib, w, d, tree, out, status) == 0
    assert tsd.launch_count() == before + 1
    torch.cuda.synchronize(dev)
    assert int(status.item()) == 0
    assert torch.equal(out.n_accepted, want.n_accepted)
    assert torch.equal(out.out_tokens, want.out_tokens)
    assert torch.equal(out.out_path, want.out_path)
    assert (out.n_accepted >= 0).all().item()
    check_stochastic(w, out, oracle.workload_stochastic(w))
