"""CPU fp64 oracle for the OneTrans block-stack forward.

TEST INFRASTRUCTURE ONLY: imported by tests/, __graft_entry__.smoke() and the
CPU-baseline legs of bench.py, never by the CUDA product path.

Parity status: every function here is pinned by the not-gpu tests (brute
force, textbook reduction, closed forms, invariants); none is unpinned.
"""
