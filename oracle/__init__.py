"""CPU oracle for the ThinKV decode hot path -- test infrastructure only.

Imported only by ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline
and reference legs of ``bench.py``; never by the CUDA library.
"""
