"""CPU oracle (test infrastructure only; see qg_oracle.py)."""
