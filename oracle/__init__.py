"""fp64 CPU oracle for zigzag ring attention.  TEST INFRASTRUCTURE ONLY.

Only tests/, __graft_entry__.smoke() and bench.py's CPU-baseline leg may import
this package.  The product package (long_sequence_context_b200) never does.
"""
