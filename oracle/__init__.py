"""Plain fp64 CPU oracle of the Gated DeltaNet recurrent-state update.

TEST INFRASTRUCTURE: only ``tests/``, ``__graft_entry__.smoke()`` and the
CPU-baseline leg of ``bench.py`` import this package. The CUDA library and its
Python binding never import it.
"""
from .gdn_oracle import Oracle, OracleF32, load, load_f32

__all__ = ["Oracle", "OracleF32", "load", "load_f32"]
