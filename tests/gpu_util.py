"""Helpers for the GPU parity tests: run the CUDA path on a Workload and
compare it with the oracle on the same seeded inputs."""

from __future__ import annotations

from typing import Dict, Optional

import numpy as np
import torch

import oracle
import tree_speculative_decoding_ancestor_b200 as tsd

# Tolerances of the attention output against the fp64 oracle (max-abs).
ATOL = {"bf16": 2e-2, "f32": 1e-4}
# Boundary-excused stochastic mismatches must stay below this fraction of draws.
EXCUSED_MAX_FRACTION = 1e-4


def to_dev(w, dev):
    """Copy every tensor field of a Workload to the device."""
    fields = ["parent", "n_nodes", "prefix_len", "tokens", "q_row", "q", "k_cache", "v_cache",
              "logits", "q_probs", "u_accept", "u_sample"]
    return {f: getattr(w, f).to(dev) for f in fields}


def run_tree(d) -> tsd.TreeMask:
    return tsd.tree_mask_build(d["parent"], d["n_nodes"])


def check_mask(w, tree: tsd.TreeMask) -> None:
    ref = oracle.tree_mask(w.parent, w.n_nodes, w.Tmax)
    mask = tree.mask.cpu().numpy().view(np.uint32)
    assert (mask == ref["mask"]).all()
    assert (tree.depth.cpu().numpy() == ref["depth"]).all()
    fc = tree.first_child.cpu().numpy()
    bad = ref["status"] != 0
    ref_fc = ref["first_child"].copy()
    ref_fc[bad, 0] = -2
    assert (fc == ref_fc).all()
    assert (tree.next_sibling.cpu().numpy() == ref["next_sibling"]).all()


def check_attention(w, got: torch.Tensor, ref: Optional[np.ndarray] = None,
                    sentinel: Optional[float] = None) -> float:
    """Max-abs error over valid rows; padding rows must still hold `sentinel`."""
    if ref is None:
        ref = oracle.workload_attention(w)
    g = got.float().cpu().numpy().astype(np.float64)
    if sentinel is not None:   # the value the sentinel has in the output's dtype
        sentinel = float(torch.tensor(sentinel, dtype=got.dtype).float())
    worst = 0.0
    for b in range(w.B):
        T = int(w.n_nodes[b])
        if T:
            err = np.abs(g[b, :T] - ref[b, :T])
            assert np.isfinite(g[b, :T]).all()
            worst = max(worst, float(err.max()))
        if sentinel is not None:
            assert (g[b, T:] == sentinel).all(), "padding rows were written"
    assert worst <= ATOL[w.dtype], f"max abs err {worst} > {ATOL[w.dtype]}"
    return worst


def check_greedy(w, res: tsd.VerifyResult, ref: Optional[Dict] = None) -> None:
    if ref is None:
        ref = oracle.workload_greedy(w)
    n = res.n_accepted.cpu().numpy()
    assert (n == ref["n_accepted"]).all(), (n, ref["n_accepted"])
    ot, op = res.out_tokens.cpu().numpy(), res.out_path.cpu().numpy()
    for b in range(w.B):
        k = int(n[b])
        if k < 0:
            continue
        assert (op[b, :k] == ref["out_path"][b, :k]).all()
        assert (ot[b, :k + 1] == ref["out_tokens"][b, :k + 1]).all()


def check_stochastic(w, res: tsd.VerifyResult, ref: Optional[Dict] = None) -> Dict[str, int]:
    """Bit-exact except sequences whose oracle path had a boundary-flagged
    decision (|u - C_i| <= 1e-9 or |u q - p| <= 1e-9 q)."""
    if ref is None:
        ref = oracle.workload_stochastic(w)
    n = res.n_accepted.cpu().numpy()
    ot, op = res.out_tokens.cpu().numpy(), res.out_path.cpu().numpy()
    mism, excused = 0, 0
    for b in range(w.B):
        k = int(ref["n_accepted"][b])
        same = int(n[b]) == k
        if same and k >= 0:
            same = (op[b, :k] == ref["out_path"][b, :k]).all() and \
                (ot[b, :k + 1] == ref["out_tokens"][b, :k + 1]).all()
        if not same:
            mism += 1
            assert ref["n_flagged"][b] > 0, f"sequence {b}: unexcused mismatch"
            excused += 1
    decisions = int(ref["n_decisions"].sum())
    assert excused <= max(0, EXCUSED_MAX_FRACTION * decisions)
    return dict(mismatches=mism, excused=excused, decisions=decisions)


def poison(w, dev_tensors, value=float("nan")):
    """Fill what the kernels must ignore: padding query rows and every cache
    position at or beyond prefix_len + n_nodes."""
    q, k, v = dev_tensors["q"], dev_tensors["k_cache"], dev_tensors["v_cache"]
    for b in range(w.B):
        T, P = int(w.n_nodes[b]), int(w.prefix_len[b])
        q[b, T:] = value
        k[b, :, P + T:] = value
        v[b, :, P + T:] = value
