"""CPU oracle for the store-h decode-attention path (test infrastructure only).

Only the tests, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package.  The product library never does.

Two implementations of the same definitions, pinned by the same tests:
``oracle.cpp`` (plain C++ loops in FP64, ``storeh_oracle.cpp``), the checker of
the GPU tests and the timed CPU baseline, and the numpy one re-exported here
(``storeh_oracle.py``), on which the tree and delta oracles build.
"""
from .storeh_oracle import *  # noqa: F401,F403
from . import delta_oracle  # noqa: F401  (iteration-axis delta cache)
from . import tree_oracle  # noqa: F401  (tree verification over the cache)
