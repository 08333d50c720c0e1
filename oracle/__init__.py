"""Plain, slow fp64 CPU oracle of the DeepSeek-Sparse-Attention step with IndexShare.

TEST INFRASTRUCTURE ONLY.  Nothing on the product path may import this package:
only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline / reference arm
of ``bench.py`` call it.  It shares no code with the CUDA library.
"""
from .dsa_oracle import *  # noqa: F401,F403
