"""CPU oracle (test infrastructure only; see flashsvd_oracle.py)."""
