"""B200-native verification hot path of tree speculative decoding (SpecInfer).

Six operations, each a thin wrapper over the C ABI of ``lib/libtsd.so``
(``include/tsd.h``):

* :func:`tree_mask_build`     -- ancestor bitmask / depth / child lists from ``parent[]``;
* :func:`tree_attention`      -- topology-aware tree attention over prefix KV + ancestors
  (:func:`tree_attention_paged` for a paged KV cache with a block table);
* :func:`tree_verify_greedy`  -- longest argmax-matching root path + one bonus token;
* :func:`tree_verify_stochastic` -- multi-step speculative sampling (exact target distribution);
* :func:`kv_commit`           -- move the accepted nodes' K/V rows after the prefix;
* :func:`tree_expand`, :func:`tree_merge_chains`, :func:`tree_dfs_order` -- build the
  token tree (expansion top-k levels, merge of several SSMs' chains, depth-first order);
* :func:`all_gather_accepted` -- with one batch per GPU, every rank's verification
  results on every rank (the batch-sharded path's only collective, optional).
"""

from .binding import (  # noqa: F401
    LIB_PATH,
    TsdError,
    Tree,
    TreeMask,
    VerifyResult,
    attention_plan,
    attention_workspace_size,
    device_status,
    exported_symbols,
    kv_commit,
    launch_count,
    load_library,
    tree_attention,
    tree_attention_paged,
    tree_dfs_order,
    tree_expand,
    tree_mask_build,
    tree_merge_chains,
    tree_verify_greedy,
    tree_verify_stochastic,
    tree_verify_stochastic_noalloc,
    verify_greedy_plan,
    verify_stochastic_plan,
    verify_workspace_size,
)
from .dist import all_gather_accepted  # noqa: F401
