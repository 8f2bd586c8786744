"""fp64 CPU oracle for the fused LoRA linear layer (test infrastructure only).

Imported only by ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline
leg of ``bench.py``; the product path never imports it.
"""
from .oracle import *  # noqa: F401,F403
