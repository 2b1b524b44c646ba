"""CPU oracle package (test infrastructure only; see sage2_oracle.py)."""
