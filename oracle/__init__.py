"""CPU oracle (test infrastructure only; see lsh_oracle.py)."""
