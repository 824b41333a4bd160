"""CPU oracle (test infrastructure): float64 numpy restatement of the attention path.

Importable only from tests/, __graft_entry__.smoke() and bench.py's CPU-baseline legs.
"""
