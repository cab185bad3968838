"""CPU float64 oracle (test infrastructure only; see park_oracle.py)."""
