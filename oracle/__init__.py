"""CPU oracle for the AB-Attention hot path (test infrastructure only).

Only tests/, __graft_entry__.smoke() and bench.py's CPU-baseline leg may import
this package; the library and its binding never do.
"""
