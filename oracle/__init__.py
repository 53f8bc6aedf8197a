"""fp64 CPU oracle for causal alpha-entmax attention (test infrastructure; see oracle.py)."""
