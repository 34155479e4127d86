"""The attention launch plan (tsd_tree_attention_plan), on the host (CPU only).

The plan names the kernel, the query-row blocks and the key-range splits
that tree_attention uses for given sizes and SM count. Pinned here for the
five workloads on a 148-SM B200 (the grids the benchmark measures), for the
environment selections, and against the workspace size (partials exist only
when the keys are split).
"""

import pytest
import torch

import tree_speculative_decoding_ancestor_b200 as tsd
from workloads import gen

SMS = 148

EXPECTED = {   # workload -> (kernel, row blocks, splits)
    "tiny": ("simt", 1, 1),
    "llama7b": ("rows64", 1, 1),
    "merge": ("rows64", 1, 1),
    "gqa70b": ("rows128", 4, 1),
    "long32k": ("rows128", 4, 8),
}


def _sizes(name):
    """Sizes of a workload from its configuration: every sequence holds the
    full prefix, and the cache ends after the tree slots."""
    c = gen.CONFIGS[gen.WORKLOAD_NAMES[name]]
    dt = torch.bfloat16 if c["dtype"] == "bf16" else torch.float32
    return (c["B"], c["Tmax"], c["Hq"], c["Hkv"], c["D"], c["P"] + c["Tmax"], dt)


def test_sizes_match_the_generated_workload():
    w = gen.config_workload(gen.WORKLOAD_NAMES["tiny"])
    assert _sizes("tiny")[:6] == (w.B, w.Tmax, w.Hq, w.Hkv, w.D, int(w.k_cache.shape[2]))


@pytest.fixture(autouse=True)
def _no_selection(monkeypatch):
    for v in ("TSD_ATTN_ROWS_VARIANT", "TSD_ATTN_SMALL_VARIANT", "TSD_FORCE_PATH"):
        monkeypatch.delenv(v, raising=False)


@pytest.mark.parametrize("name", sorted(EXPECTED))
def test_plan_of_each_workload(name):
    B, Tmax, Hq, Hkv, D, Lmax, dt = _sizes(name)
    p = tsd.attention_plan(B, Tmax, Hq, Hkv, D, Lmax, dt, SMS)
    assert (p["kernel"], p["row_blocks"], p["splits"]) == EXPECTED[name]
    # the splits cover the keys
    assert p["splits"] * p["keys_per_split"] >= Lmax
    assert (p["splits"] - 1) * p["keys_per_split"] < Lmax
    # partial results (workspace) exist exactly when the keys are split
    # (the workspace query sizes for the current device: 148 SMs without one)
    if p["kernel"] != "simt":
        ws = tsd.attention_workspace_size(B, Tmax, Hq, Hkv, D, Lmax, dt)
        assert (ws > 0) == (p["splits"] > 1)


def test_environment_selects_the_other_kernels(monkeypatch):
    monkeypatch.setenv("TSD_ATTN_ROWS_VARIANT", "2")
    assert tsd.attention_plan(*_sizes("gqa70b"), SMS)["kernel"] == "rows64"
    monkeypatch.setenv("TSD_ATTN_SMALL_VARIANT", "keysplit")
    assert tsd.attention_plan(*_sizes("merge"), SMS)["kernel"] == "keysplit"
    monkeypatch.setenv("TSD_FORCE_PATH", "simt")
    assert tsd.attention_plan(*_sizes("gqa70b"), SMS)["kernel"] == "simt"


def test_more_splits_on_fewer_blocks():
    # one sequence of a long prefix: few (b, KV head) pairs, so the keys are
    # split to fill the SMs
    p = tsd.attention_plan(1, 64, 64, 8, 128, 32768 + 64, torch.bfloat16, SMS)
    assert p["kernel"] == "rows128" and p["row_blocks"] == 4 and p["splits"] >= 4


def test_plan_rejects_bad_sizes():
    with pytest.raises(tsd.TsdError):
        tsd.attention_plan(2, 8, 6, 4, 128, 64, torch.bfloat16, SMS)   # Hq % Hkv
    with pytest.raises(tsd.TsdError):
        tsd.attention_plan(2, 8, 8, 2, 96, 64, torch.bfloat16, SMS)    # head dim
    with pytest.raises(tsd.TsdError):
        tsd.attention_plan(2, 8, 8, 2, 128, 64, torch.bfloat16, 0)     # no SMs


def test_forced_split_count(monkeypatch):
    B, Tmax, Hq, Hkv, D, Lmax, dt = _sizes("llama7b")
    monkeypatch.setenv("TSD_ATTN_SPLITS", "3")
    p = tsd.attention_plan(B, Tmax, Hq, Hkv, D, Lmax, dt, SMS)
    assert p["kernel"] == "rows64" and p["splits"] == 3
    assert 3 * p["keys_per_split"] >= Lmax and p["keys_per_split"] % 64 == 0
    # the partial results are sized for the forced splits
    assert tsd.attention_workspace_size(B, Tmax, Hq, Hkv, D, Lmax, dt) > 0
    monkeypatch.setenv("TSD_ATTN_SPLITS", "1000")     # clamped to one split per key tile
    p = tsd.attention_plan(B, Tmax, Hq, Hkv, D, Lmax, dt, SMS)
    assert p["splits"] == (Lmax + 63) // 64
    monkeypatch.setenv("TSD_ATTN_SPLITS", "4")        # the CUDA-core path: 128 keys at least
    assert tsd.attention_plan(*_sizes("tiny"), SMS)["splits"] == 1


def test_greedy_form_follows_the_scan_size(monkeypatch):
    # the walk over matched nodes for batches whose logits reach 64 MiB (the
    # 70B-GQA workload: 32 x 65 rows x 32000), the all-rows scan below
    # (LLaMA-7B: 8 x 21 rows); TSD_GREEDY_FORM forces either
    monkeypatch.delenv("TSD_GREEDY_FORM", raising=False)
    assert tsd.verify_greedy_plan(32, 64, 32000)["form"] == "walk"
    assert tsd.verify_greedy_plan(8, 20, 32000)["form"] == "rows"
    rows = 64 * 1024 * 1024 // (4 * 32000)          # rows of 64 MiB at V = 32000
    assert tsd.verify_greedy_plan(1, 127, 32000)["form"] == "rows"   # 128 rows
    assert tsd.verify_greedy_plan(rows // 128 + 1, 127, 32000)["form"] == "walk"
    monkeypatch.setenv("TSD_GREEDY_FORM", "walk")
    assert tsd.verify_greedy_plan(1, 6, 32)["form"] == "walk"
    monkeypatch.setenv("TSD_GREEDY_FORM", "rows")
    assert tsd.verify_greedy_plan(32, 64, 32000)["form"] == "rows"
    with pytest.raises(tsd.TsdError):
        tsd.verify_greedy_plan(0, 6, 32)
