"""Plain fp64 CPU oracle for the compressed KV-cache path.

TEST INFRASTRUCTURE ONLY.  Nothing in the product path may import, call or
execute this package: only ``tests/``, ``__graft_entry__.smoke()`` and the
``cpu_baseline`` / ``--impl reference`` legs of ``bench.py`` use it.  It shares
no code with the CUDA library (no kernels, headers, tables or constant
generators); the only thing both sides consume is the seeded input generator
module, which holds none of the method's arithmetic.

Modules
-------
``tq_oracle``  vectorised NumPy float64 implementation of the format and of
               decode attention / eviction / inner-product search.
``brute``      the same definitions as explicit pure-Python loops, for tiny
               sizes; it exists to cross-check ``tq_oracle``.
"""
