"""fp64 CPU oracle for MLA paged decoding.

Test infrastructure only: imported by tests/, __graft_entry__.smoke() and the
CPU-baseline / reference legs of bench.py, never by the CUDA path.
"""
