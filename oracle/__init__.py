"""fp64 CPU oracle of the performer unit step.

TEST INFRASTRUCTURE: only ``tests/``, ``__graft_entry__.smoke()`` and the
CPU-baseline legs of ``bench.py`` may import it.  The CUDA library never does.
"""
