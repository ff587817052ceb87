"""fp64 CPU oracle for MLA decode (test infrastructure only).

Only ``tests/``, ``__graft_entry__.smoke()`` and ``bench.py``'s CPU-baseline leg
import this package.  The CUDA library never does, and this package imports
nothing from it.
"""
