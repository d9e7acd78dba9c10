"""CPU oracle (test infrastructure only; see hca_oracle.py)."""
