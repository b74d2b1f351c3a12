"""fp64 CPU oracle (test infrastructure only; see sbp_oracle.py)."""
