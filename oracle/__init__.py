"""CPU oracle for the store-h decode-attention path (test infrastructure only).

Only the tests, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package.  The product library never does.
"""
from .storeh_oracle import *  # noqa: F401,F403
from . import delta_oracle  # noqa: F401  (iteration-axis delta cache)
from . import tree_oracle  # noqa: F401  (tree verification over the cache)
