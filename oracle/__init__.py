"""Float64 CPU oracle for the VDA linear branch -- test infrastructure only.

Only tests/, __graft_entry__.smoke() and bench.py's CPU-baseline leg import it.
"""
