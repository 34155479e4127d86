"""The Python binding's argument checks (CPU only).

Every entry point checks each tensor it hands to the library (device,
dtype, shape, contiguity), including caller-supplied outputs, tree arrays,
workspaces and status words. An output of the wrong size would otherwise be
written past its end on the GPU. Here the library is replaced by a stand-in
that records the calls and succeeds, and the CUDA-only pieces are stubbed,
so the checks run on CPU tensors: valid arguments must reach the library,
and invalid ones must be refused before it.
"""

import pytest
import torch

import tree_speculative_decoding_ancestor_b200 as tsd
from tree_speculative_decoding_ancestor_b200 import binding


class _Lib:
    def __init__(self):
        self.calls = []

    def __getattr__(self, name):
        def call(*args):
            self.calls.append(name)
            return 0
        return call


@pytest.fixture
def lib(monkeypatch):
    fake = _Lib()
    monkeypatch.setattr(binding, "load_library", lambda *a: fake)
    monkeypatch.setattr(binding, "_cuda", lambda dev: None)
    monkeypatch.setattr(binding, "_stream", lambda dev: 0)
    st = torch.zeros(1, dtype=torch.int32)
    monkeypatch.setattr(binding, "device_status", lambda dev=None: st)
    return fake


B, Tmax, V, Hq, Hkv, D, L = 2, 8, 50, 4, 2, 64, 40
i32 = dict(dtype=torch.int32)


def _tree():
    return tsd.TreeMask(torch.zeros(B, Tmax, 1, **i32), torch.zeros(B, Tmax, **i32),
                        torch.zeros(B, Tmax + 1, **i32), torch.zeros(B, Tmax, **i32))


def _result(T=Tmax):
    return tsd.VerifyResult(torch.zeros(B, T + 1, **i32), torch.zeros(B, T, **i32),
                            torch.zeros(B, **i32))


def _verify_args():
    return dict(logits=torch.zeros(B, Tmax + 1, V), tokens=torch.zeros(B, Tmax, **i32),
                n_nodes=torch.zeros(B, **i32))


def _stochastic(out=None, tree=None, **kw):
    a = _verify_args()
    return tsd.tree_verify_stochastic(
        a["logits"], 1.0, torch.zeros(B, 3, V), torch.zeros(B, Tmax, **i32), a["tokens"],
        a["n_nodes"], tree or _tree(), torch.full((B, Tmax), 0.5, dtype=torch.float64),
        torch.full((B, Tmax + 1), 0.5, dtype=torch.float64), out=out, **kw)


def test_valid_calls_reach_the_library(lib):
    parent = torch.full((B, Tmax), -1, **i32)
    n = torch.zeros(B, **i32)
    tree = tsd.tree_mask_build(parent, n)
    tsd.tree_mask_build(parent, n, out=_tree())
    q = torch.zeros(B, Tmax, Hq, D, dtype=torch.bfloat16)
    kv = torch.zeros(B, Hkv, L, D, dtype=torch.bfloat16)
    tsd.tree_attention(q, kv, kv, n, n, tree.mask)
    tsd.tree_attention(q, kv, kv, n, n, tree.mask, out=torch.empty_like(q),
                       workspace=torch.empty(4096, dtype=torch.uint8),
                       status=torch.zeros(1, **i32))
    a = _verify_args()
    tsd.tree_verify_greedy(a["logits"], a["tokens"], parent, a["n_nodes"], tree)
    tsd.tree_verify_greedy(a["logits"], a["tokens"], parent, a["n_nodes"], tree, out=_result())
    _stochastic()
    _stochastic(out=_result())
    pages = torch.zeros(6, Hkv, 16, D, dtype=torch.bfloat16)
    tsd.tree_attention_paged(q, pages, pages, torch.zeros(B, 3, **i32), n, n, tree.mask)
    tsd.kv_commit(kv, kv, n, _result())
    t = tsd.Tree(parent.clone(), torch.zeros(B, Tmax, **i32), torch.zeros(B, Tmax, **i32), n)
    tsd.tree_expand(torch.zeros(B, 9, V), torch.zeros(B, Tmax, **i32), 2, t, n.clone())
    tsd.tree_dfs_order(t)
    tsd.tree_merge_chains(torch.zeros(B, 3, 4, **i32), torch.zeros(B, 3, 4, **i32),
                          torch.zeros(B, 3, **i32), Tmax)
    assert lib.calls.count("tsd_tree_verify_stochastic") == 2
    assert "tsd_tree_attention_paged" in lib.calls and "tsd_tree_merge_chains" in lib.calls


def test_outputs_and_trees_of_the_wrong_size_are_refused(lib):
    parent = torch.full((B, Tmax), -1, **i32)
    n = torch.zeros(B, **i32)
    short = _tree()._replace(first_child=torch.zeros(B, Tmax, **i32))   # needs Tmax + 1
    with pytest.raises(ValueError):
        tsd.tree_mask_build(parent, n, out=short)
    a = _verify_args()
    with pytest.raises(ValueError):
        tsd.tree_verify_greedy(a["logits"], a["tokens"], parent, a["n_nodes"], short)
    with pytest.raises(ValueError):   # an output sized for a smaller tree
        tsd.tree_verify_greedy(a["logits"], a["tokens"], parent, a["n_nodes"], _tree(),
                               out=_result(Tmax - 1))
    with pytest.raises(ValueError):
        _stochastic(out=_result(Tmax - 1))
    with pytest.raises(ValueError):
        _stochastic(tree=_tree()._replace(next_sibling=torch.zeros(B, Tmax - 1, **i32)))
    with pytest.raises(TypeError):    # int64 where int32 is read
        _stochastic(out=_result()._replace(n_accepted=torch.zeros(B, dtype=torch.int64)))
    noncontig = torch.zeros(Tmax + 1, B, **i32).t()
    with pytest.raises(ValueError):
        _stochastic(out=_result()._replace(out_tokens=noncontig))
    assert not any(c.startswith("tsd_tree_verify") or c == "tsd_tree_mask_build"
                   for c in lib.calls)


def test_workspace_and_status_must_fit(lib):
    parent = torch.full((B, Tmax), -1, **i32)
    n = torch.zeros(B, **i32)
    tree = tsd.tree_mask_build(parent, n)
    q = torch.zeros(B, Tmax, Hq, D, dtype=torch.bfloat16)
    kv = torch.zeros(B, Hkv, L, D, dtype=torch.bfloat16)
    with pytest.raises(TypeError):    # element count would not be the byte count
        tsd.tree_attention(q, kv, kv, n, n, tree.mask, workspace=torch.empty(64))
    with pytest.raises(ValueError):
        tsd.tree_attention(q, kv, kv, n, n, tree.mask, status=torch.zeros(1))
    with pytest.raises(ValueError):
        tsd.tree_mask_build(parent, n, status=torch.zeros(0, **i32))


def test_host_tensors_are_refused_before_the_library():
    # without the stubs: CPU tensors never reach a launch
    parent = torch.full((B, Tmax), -1, **i32)
    with pytest.raises(ValueError, match="CUDA device"):
        tsd.tree_mask_build(parent, torch.zeros(B, **i32))
    q = torch.zeros(B, Tmax, Hq, D, dtype=torch.bfloat16)
    with pytest.raises(ValueError, match="CUDA device"):
        tsd.tree_attention(q, q, q, parent[:, 0], parent[:, 0], parent)


def test_cached_workspaces_are_per_stream(lib, monkeypatch):
    # Calls without a workspace on two streams must not share a buffer (their
    # kernels may overlap); calls on one stream reuse the same buffer.
    monkeypatch.setattr(binding, "_workspace", {})
    dev = torch.device("cpu")
    seen = {}
    for handle in (11, 22, 11):
        monkeypatch.setattr(binding, "_stream", lambda d, h=handle: h)
        ws = binding._workspace_for(dev, "verify", 512, None)
        assert ws.numel() >= 512
        seen.setdefault(handle, []).append(ws.data_ptr())
    assert seen[11][0] == seen[11][1]
    assert seen[11][0] != seen[22][0]
    # through an entry point: the stochastic verifier on two streams
    bufs = []
    for handle in (33, 44):
        monkeypatch.setattr(binding, "_stream", lambda d, h=handle: h)
        _stochastic()
        bufs.append(binding._workspace[(None, "verify", handle)].data_ptr())
    assert bufs[0] != bufs[1]
