"""fp64 CPU oracle for exact attention -- test infrastructure only.

Only tests/, __graft_entry__.smoke() and bench.py's CPU-baseline leg may
import this package; the CUDA path never does.
"""
