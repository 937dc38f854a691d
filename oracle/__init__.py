"""CPU oracle for the MSA hot path (test infrastructure only; see oracle.py)."""
