"""CPU oracle: test infrastructure only (see nf4_oracle.py)."""
