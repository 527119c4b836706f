"""fp64 CPU oracle of the TTT-MLP layer scan (test infrastructure only).

Importable only from tests/, __graft_entry__.smoke() and bench.py's CPU
baseline leg; the CUDA library never uses it.
"""
