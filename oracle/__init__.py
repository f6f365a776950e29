"""fp64 CPU oracle of SAS gated block-sparse attention (test infrastructure).

Only tests/, __graft_entry__.smoke() and bench.py's CPU arm use this package;
the library's CUDA path never imports or calls it.
"""
