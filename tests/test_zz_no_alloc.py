"""The allocation-free stochastic verifier (tsd_tree_verify_stochastic_noalloc).

Some callers cannot hand the library a scratch buffer: a serving engine whose
KV-cache pool already owns nearly all device memory, or a caller that reaches
the library through a plain C interface with no device allocator.  This entry
point keeps its scratch in a fixed array inside the library instead.  These
tests call it through the C ABI (ctypes, no Python wrapper in between) and
check that it returns exactly what the workspace entry point returns, on two
calls in a row (the second call finds the first call's leftovers in the
shared array), and that oversize problems are refused without a launch.

This file is collected last on purpose, so that a run stopping at the first
failure has already run every other test.
"""

import ctypes

import pytest
import torch

import tree_speculative_decoding_ancestor_b200 as tsd
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
    assert int(status.item()) == 0


def test_noalloc_refuses_oversize(cuda_device):
    lib = tsd.load_library()
    # B * (Tmax + 1) = 90300 logits rows needs ~2.5 MB of scratch, more than
    # the fixed 1 MiB.  Real tensors of that shape (tiny vocabulary, empty
    # trees) keep every pointer valid for the sizes passed.
    B, Tmax, V = 700, 128, 4
    dev = cuda_device
    i32 = lambda *s: torch.zeros(s, dtype=torch.int32, device=dev)  # noqa: E731
    d = {"logits": torch.zeros((B, Tmax + 1, V), dtype=torch.float32, device=dev),
         "q_probs": torch.full((B, 1, V), 0.25, dtype=torch.float32, device=dev),
         "q_row": i32(B, Tmax), "tokens": i32(B, Tmax), "n_nodes": i32(B),
         "u_accept": torch.full((B, Tmax), 0.5, dtype=torch.float64, device=dev),
         "u_sample": torch.full((B, Tmax + 1), 0.5, dtype=torch.float64, device=dev)}
    tree = tsd.tree_mask_build(torch.full((B, Tmax), -1, dtype=torch.int32, device=dev),
                               d["n_nodes"])

    class W:
        temperature = 1.0
    W.B, W.Tmax, W.V = B, Tmax, V
    status = torch.zeros(1, dtype=torch.int32, device=dev)
    out = _outputs(B, Tmax, dev)
    torch.cuda.synchronize(dev)
    before = tsd.launch_count()
    assert _call_noalloc(lib, W, d, tree, out, status) == TSD_ERR_WORKSPACE
    assert tsd.launch_count() == before
    torch.cuda.synchronize(dev)
    assert (out.n_accepted == -7).all().item()
    # the workspace entry point handles the same problem
    res = tsd.tree_verify_stochastic(d["logits"], 1.0, d["q_probs"], d["q_row"], d["tokens"],
                                     d["n_nodes"], tree, d["u_accept"], d["u_sample"])
    assert (res.n_accepted == 0).all().item()
