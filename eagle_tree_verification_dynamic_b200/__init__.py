"""B200-native EAGLE tree-verification step.

The compute lives in ``libeagle_tree.so`` (CUDA, sm_100a) behind the C ABI in
``include/eagle_tree.h``; this package is its thin Python binding.  Importing
the package does not load the library; the first call does, and raises
``EagleError`` if the library has not been built.
"""
from ._lib import (  # noqa: F401
    BF16,
    F32,
    EagleError,
    Tree,
    TreeGrower,
    accept,
    accept_into,
    accept_workspace_bytes,
    alloc_tree,
    attention_workspace_bytes,
    exported_names,
    kv_compact,
    kv_compact_paged,
    kv_compact_paged_into,
    tree_attention_paged,
    tree_attention_paged_into,
    static_tree_build,
    static_tree_rows,
    kv_compact_into,
    lib,
    pool_size,
    step_in,
    step_into,
    step_workspace_bytes,
    row_stats,
    tree_attention,
    tree_attention_into,
    tree_build,
    tree_build_into,
    tree_build_workspace_bytes,
    tree_mask,
    tree_mask_into,
)
