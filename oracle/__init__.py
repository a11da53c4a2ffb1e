"""CPU oracle for the packed-tree SSM scan -- TEST INFRASTRUCTURE ONLY.

Only the tests, ``__graft_entry__.smoke()`` and the benchmark's CPU-baseline leg
may import this package.  The CUDA library and its Python binding never import,
load or call it, and the two share no code.

* ``walk``   -- the plain definition: a fp64 C walk of every node's root path
               (``stree_oracle.c``), wrapped with ctypes.
* ``packed`` -- a second fp64 formulation (numpy) of the same outputs through the
               accumulated transition ``A_tree = L . log A``; used only to
               cross-check the walk.
* ``accept`` -- verification of the draft tree: greedy (temperature 0) and by
               multi-step speculative sampling; the accepted path and bonus token.
* ``attention`` -- tree-masked attention of the hybrid model's Transformer layers
               over the packed tree (context plus each node's root path).
* ``gdn``    -- the gated delta rule (linear-attention layers) over the packed tree:
               the root-path walk, its commit, and a packed cross-check.
"""
from .walk import (  # noqa: F401
    build_oracle,
    oracle_build_tree,
    oracle_commit,
    oracle_max_threads,
    oracle_tree_scan,
)
from .accept import oracle_accept_greedy, oracle_accept_sampling  # noqa: F401,E402
from .attention import oracle_tree_attention  # noqa: F401,E402
from .gdn import oracle_gdn_commit, oracle_gdn_tree  # noqa: F401,E402
