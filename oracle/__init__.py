"""fp64 CPU oracle for the DSA hot path -- TEST INFRASTRUCTURE ONLY.

Only ``tests/``, ``__graft_entry__.smoke()`` and ``bench.py``'s CPU-baseline leg may
import it.  The CUDA library never imports it, and it never imports the CUDA library.
"""
