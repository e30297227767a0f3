"""CPU oracle (test infrastructure only; see hsq_oracle.py)."""
