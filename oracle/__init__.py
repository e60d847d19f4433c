"""fp64 CPU oracle for block-causal GQA attention with QK-RMSNorm.

TEST INFRASTRUCTURE ONLY: imported by ``tests/``, ``__graft_entry__.smoke()``
and ``bench.py``'s CPU-baseline / reference legs, never by the product path.
"""
from .bca_oracle import *  # noqa: F401,F403
from .bca_oracle import __all__  # noqa: F401
