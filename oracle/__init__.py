"""fp64 CPU oracle for the VDN-H3 dual-branch hybrid attention.

TEST INFRASTRUCTURE ONLY: imported by ``tests/``, ``__graft_entry__.smoke()``
and the CPU-baseline leg of ``bench.py``; never by the product path.
Modules: :mod:`oracle.hybrid_attn` (the definition, step by step) and
:mod:`oracle.bruteforce` (independent formulations that pin it).
"""
