"""Small cases of every kernel on the bounds-checked debug build.

Run as a script in a process of its own with TSD_LIBRARY pointing at
lib/libtsd_checked.so (tests/test_gpu_checked_build.py does that): the
library is chosen at its first load.  Every case is compared with the oracle
as in the parity tests, and the status word must end with no bit set -- in
particular not TSD_DEV_BOUNDS, which the checked build raises for an index
outside its buffer.  Prints "checked ok" at the end.
"""

import os
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, os.path.dirname(HERE))
sys.path.insert(0, HERE)

import torch  # noqa: E402

import oracle  # noqa: E402
import tree_speculative_decoding_ancestor_b200 as tsd  # noqa: E402
from gpu_util import (check_attention, check_greedy, check_mask, check_stochastic,  # noqa: E402
                      poison, run_tree, to_dev)
from workloads import gen  # noqa: E402


def main():
    assert tsd.LIB_PATH.endswith("libtsd_checked.so"), tsd.LIB_PATH
    dev = torch.device("cuda:0")
    st = tsd.device_status(dev)
    kernels = [{}, {"TSD_ATTN_SOFTMAX_WARPS": "2"}, {"TSD_ATTN_ROWS_VARIANT": "2"},
               {"TSD_ATTN_SMALL_VARIANT": "keysplit"}, {"TSD_FORCE_PATH": "simt"}]
    shapes = [dict(seed=3, B=3, Tmax=24, Hq=16, Hkv=2, D=128, P_max=513),    # 192 rows
              dict(seed=4, B=2, Tmax=20, Hq=8, Hkv=2, D=128, P_max=300),     # 80 rows
              dict(seed=5, B=2, Tmax=9, Hq=4, Hkv=4, D=64, P_max=70, dtype="f32")]
    for shape in shapes:
        c = dict(shape)
        w = gen.random_workload(c.pop("seed"), max_children=4, max_depth=10, lmax_pad=13,
                                V=700, **{"dtype": "bf16", **c})
        d = to_dev(w, dev)
        poison(w, d)
        tree = run_tree(d)
        check_mask(w, tree)
        ref = oracle.workload_attention(w)
        for env in kernels:
            for splits in ("1", "3"):
                os.environ.update(env)
                os.environ["TSD_ATTN_SPLITS"] = splits
                out = torch.full_like(d["q"], 1234.0)
                tsd.tree_attention(d["q"], d["k_cache"], d["v_cache"], d["prefix_len"],
                                   d["n_nodes"], tree.mask, out=out)
                check_attention(w, out, ref=ref, sentinel=1234.0)
                for k in env:
                    del os.environ[k]
                del os.environ["TSD_ATTN_SPLITS"]
        for form in ("walk", "rows"):   # both greedy forms
            os.environ["TSD_GREEDY_FORM"] = form
            check_greedy(w, tsd.tree_verify_greedy(d["logits"], d["tokens"], d["parent"],
                                                   d["n_nodes"], tree))
        del os.environ["TSD_GREEDY_FORM"]
        check_stochastic(w, tsd.tree_verify_stochastic(
            d["logits"], w.temperature, d["q_probs"], d["q_row"], d["tokens"], d["n_nodes"],
            tree, d["u_accept"], d["u_sample"]))
        res = oracle.workload_greedy(w)
        path = tsd.VerifyResult(torch.zeros_like(d["tokens"]),
                                torch.from_numpy(res["out_path"]).to(dev),
                                torch.from_numpy(res["n_accepted"]).to(dev))
        tsd.kv_commit(d["k_cache"], d["v_cache"], d["prefix_len"], path)
    torch.cuda.synchronize(dev)
    assert int(st.item()) == 0, f"status word {int(st.item())}"
    print("checked ok")


if __name__ == "__main__":
    main()
