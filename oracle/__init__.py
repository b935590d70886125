"""Float64 CPU oracle for remapped-RoPE causal attention.

TEST INFRASTRUCTURE ONLY. Nothing on the product path imports this package:
only the tests, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may use it. It shares no code with the CUDA library.
"""
from .ref import *  # noqa: F401,F403
