"""hybrid_packed_tree_b200 -- packed-tree selective-SSM scan on B200 (sm_100a).

The scan verifies a whole speculative draft tree in one pass and a commit step
replays the accepted root->leaf path into the new cached state ("STree:
Speculative Tree Decoding for Hybrid State Space Models", section "Approach").

* ``hybrid_packed_tree_b200.stree``     -- thin ctypes binding of ``libstree.so``
  (the C-ABI in ``include/stree.h``); importing it loads the CUDA library and
  fails loudly when it is missing.
* ``hybrid_packed_tree_b200.workloads`` -- seeded synthetic inputs.
* ``hybrid_packed_tree_b200.build``     -- nvcc build of ``libstree.so``.

Nothing is imported eagerly, so the input generator can be used without CUDA.
"""
__all__ = ["stree", "workloads", "build"]
