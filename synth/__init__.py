"""Seeded synthetic inputs for tree verification.

This package only draws random inputs (tree shapes, query/key/value tensors,
target and draft logits, draft distributions, child tokens).  It holds none of
the verification arithmetic: the CUDA library and the fp64 oracle both consume
the arrays it returns, and neither imports the other.
"""

from .workloads import (  # noqa: F401
    CONFIGS,
    AttnCase,
    AcceptCase,
    ExpandCase,
    tree_binary,
    tree_chain,
    tree_star,
    tree_bfs_fanout,
    tree_random_depth_limited,
    tree_random_recursive,
    config_tree,
    config_prefix_lens,
    tree_depths,
    attn_case,
    accept_case,
    expand_case,
    config_attn_case,
    config_accept_case,
    config_expand_case,
)
