"""fp64 CPU oracle for the ClusterAttention forward path.

TEST INFRASTRUCTURE ONLY. Only ``tests/``, ``__graft_entry__.smoke()`` and the
CPU-baseline leg of ``bench.py`` may import this package. The product path
(the ``free_clustered_block_b200`` package and its CUDA library) never does.
"""
from .ca_oracle import *  # noqa: F401,F403
