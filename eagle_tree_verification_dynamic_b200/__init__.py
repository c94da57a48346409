"""B200-native EAGLE tree-verification step.

The compute lives in ``libeagle_tree.so`` (CUDA, sm_100a) behind the C ABI in
``include/eagle_tree.h``; this package is its thin Python binding.  Importing
the package does not load the library; the first call does, and raises
``EagleError`` if the library has not been built.

One step, call by call (device tensors; ``*_into`` variants write into
preallocated outputs and workspaces, for CUDA-graph capture):

* ``tree_build``       EAGLE-2 dynamic tree from the draft rows
  (``TreeGrower`` builds the same tree one level at a time;
  ``static_tree_build`` fills EAGLE-1's fixed template instead)
* ``tree_mask``        ancestor bitmask and position ids
* ``tree_attention``   tree-masked attention over the prefix cache and the tree
  (``tree_attention_paged`` for a paged cache)
* ``accept``           greedy or sampled acceptance, with or without replacement
* ``kv_compact``       the accepted path's keys and values into the cache
  (``kv_compact_paged``)

``step.VerifyStep`` runs the whole step with preallocated buffers, as separate
calls or as the single fused ``eagle_verify_step``; ``sizing`` holds the
cost-aware sizing harness and ``calibrate`` measures its cost table.
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
    attention_wait_probe,
    attention_workspace_bytes,
    check_attention_status,
    exported_names,
    kv_compact,
    kv_compact_into,
    kv_compact_paged,
    kv_compact_paged_into,
    lib,
    pool_size,
    row_stats,
    static_template_from_paths,
    static_tree_build,
    static_tree_rows,
    step_in,
    step_into,
    step_workspace_bytes,
    tree_attention,
    tree_attention_into,
    tree_attention_paged,
    tree_attention_paged_into,
    tree_build,
    tree_build_into,
    tree_build_workspace_bytes,
    tree_mask,
    tree_mask_into,
)
