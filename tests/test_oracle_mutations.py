"""Plant plausible mistakes in the oracle and check that its pins catch them
(CPU only).

Each case copies oracle/tsd_oracle.c, applies one textual change that a
careless implementation of the pages could contain, compiles the copy, routes
the oracle through it and runs the pin that should fail.  A mutation that no
pin detects would mean the oracle is not pinned where it matters.
"""

import pytest

import oracle
import test_oracle_attention as pa
import test_oracle_commit as pc
import test_oracle_greedy as pg
import test_oracle_mask as pm
import test_oracle_stochastic as ps
import test_oracle_tree_build as pt

MUTATIONS = {
    # attention (SpecInfer explainer, "トークンツリー構造の仕組み")
    "prefix_not_attended": ("int P = prefix_len[b];", "int P = 0;",
                            lambda: pa.test_chain_equals_causal_attention("f32", 4)),
    "node_not_in_own_S_u": ("int n = P + np;", "int n = P + np - 1;",
                            pa.test_single_node_is_decode_attention),
    "gqa_head_mapping": ("int G = Hq / Hkv, hk = h / G;", "int G = Hq / Hkv, hk = h % Hkv;",
                         lambda: pa.test_chain_equals_causal_attention("bf16", 4)),
    "softmax_scale_dropped": ("s *= scale;", "s *= 1.0;",
                              lambda: pa.test_every_node_is_causal_attention_over_its_path(0)),
    "value_of_wrong_position": ("size_t voff = (kvbase + pos) * D;",
                                "size_t voff = (kvbase + (pos > 0 ? pos - 1 : 0)) * D;",
                                lambda: pa.test_every_node_is_causal_attention_over_its_path(1)),
    # ancestor mask
    "depth_off_by_one": ("dp[u] = d;", "dp[u] = d - 1;",
                         lambda: pm.test_mask_vs_subtree_enumeration(4)),
    "mask_misses_self": ("for (int v = u; v >= 0; v = par[v]) {\n                mk",
                         "for (int v = par[u]; v >= 0; v = par[v]) {\n                mk",
                         pm.test_merge_diagram_golden),
    # greedy (ツリー検証アルゴリズム, greedy)
    "argmax_ties_to_highest": ("if (l[i] > l[best])", "if (l[i] >= l[best])",
                               lambda: [pg.test_greedy_vs_exhaustive_search(s) for s in range(8)]),
    "greedy_ignores_ancestors": ("int parent_ok = p < 0 ? 1 : matched[p];", "int parent_ok = 1;",
                                 lambda: [pg.test_greedy_vs_exhaustive_search(s)
                                          for s in range(8)]),
    "greedy_first_not_longest": ("if (matched[u] && len[u] > best_len) {",
                                 "if (matched[u] && best < 0) {",
                                 lambda: [pg.test_greedy_vs_exhaustive_search(s)
                                          for s in range(8)]),
    # stochastic (ツリー検証アルゴリズム, P_accept and P_residual)
    "no_residual_update": ("if (S > 0.0)\n", "if (0)\n",
                           lambda: ps.test_exact_enumeration_equals_target(16, 2, 1.0)),
    "residual_not_normalised": ("p[i] = (r > 0.0 ? r : 0.0) / S;", "p[i] = (r > 0.0 ? r : 0.0);",
                                lambda: ps.test_exact_enumeration_equals_target(6, 3, 0.7)),
    "accept_ignores_ssm_prob": ("if (px > 0.0 && u * qx <= px) {", "if (px > 0.0 && u <= px) {",
                                lambda: ps.test_exact_enumeration_equals_target(16, 1, 1.3)),
    "temperature_ignored": ("- m) / temperature)", "- m) / 1.0)",
                            lambda: ps.test_no_tree_draw_is_inverse_cdf(0.5)),
    "child_uses_root_row": ("int row = cur + 1;", "int row = 0;", ps.test_chi_square_depth_two),
    # commit of the accepted path
    "commit_ignores_prefix": ("base + (size_t)(P + path[i]) * row_bytes", "base + (size_t)(path[i]) * row_bytes",
                              lambda: pc.test_commit_then_decode_equals_tree_attention(1, "bf16")),
    # tree construction
    "topk_ties_to_higher_id": ("return v > w || (v == w && i < j);", "return v > w || (v == w && i > j);",
                               pt.test_topk_ties_take_the_lower_token_id),
    "merge_never_shares": ("if (tp[v] == cur && tt[v] == t) {", "if (0) {",
                           pt.test_merge_rebuilds_the_page_figure),
    "dfs_children_reversed": ("for (int v = T - 1; v > u; --v)", "for (int v = u + 1; v < T; ++v)",
                              lambda: pt.test_dfs_order_is_the_recursive_preorder(0)),
    "commit_reverses_order": ("memcpy(base + (size_t)(P + i) * row_bytes", "memcpy(base + (size_t)(P + n - 1 - i) * row_bytes",
                              lambda: pc.test_committed_rows_follow_the_verified_tokens_in_order("greedy")),
}


@pytest.mark.parametrize("name", sorted(MUTATIONS))
def test_pin_catches_mutation(name, tmp_path):
    old, new, pin = MUTATIONS[name]
    src = oracle.source()
    assert src.count(old) >= 1, f"mutation anchor not found: {old!r}"
    lib = oracle.build_variant(src.replace(old, new), str(tmp_path / f"{name}.so"))
    with oracle.use_library(lib):
        with pytest.raises(AssertionError):
            pin()


def test_unmutated_source_passes_the_same_pins(tmp_path):
    lib = oracle.build_variant(oracle.source(), str(tmp_path / "same.so"))
    with oracle.use_library(lib):
        pa.test_chain_equals_causal_attention("f32", 4)
        pm.test_mask_vs_subtree_enumeration(4)
        pg.test_greedy_vs_exhaustive_search(0)
        ps.test_exact_enumeration_equals_target(16, 2, 1.0)


# The paged-KV gather is Python (numpy) code in the oracle package: plant the
# mistakes in a copy of its source and route the oracle through the copy.
import inspect  # noqa: E402

import test_oracle_paged as pp  # noqa: E402

PY_MUTATIONS = {
    "paged_table_ignored": ("pg = int(bt[b, j])", "pg = j"),
    "paged_row_offset": ("k[b, :, lo:hi] = kp[pg, :, :hi - lo]",
                         "k[b, :, lo:hi] = kp[pg, :, ::-1][:, :hi - lo]"),
    "paged_values_from_keys": ("v[b, :, lo:hi] = vp[pg, :, :hi - lo]",
                               "v[b, :, lo:hi] = kp[pg, :, :hi - lo]"),
}


@pytest.mark.parametrize("name", sorted(PY_MUTATIONS))
def test_paged_pin_catches_mutation(name, monkeypatch):
    old, new = PY_MUTATIONS[name]
    src = inspect.getsource(oracle.gather_pages)
    assert src.count(old) == 1, f"mutation anchor not found: {old!r}"
    ns = {}
    exec(compile(src.replace(old, new), "<mutated gather_pages>", "exec"), vars(oracle).copy(),
         ns)
    monkeypatch.setattr(oracle, "gather_pages", ns["gather_pages"])
    with pytest.raises(AssertionError):
        pp.test_paged_equals_contiguous(31, "bf16", 16)


def test_unmutated_paged_copy_passes_the_pin(monkeypatch):
    ns = {}
    exec(compile(inspect.getsource(oracle.gather_pages), "<copied gather_pages>", "exec"),
         vars(oracle).copy(), ns)
    monkeypatch.setattr(oracle, "gather_pages", ns["gather_pages"])
    pp.test_paged_equals_contiguous(31, "bf16", 16)
