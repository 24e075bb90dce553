"""Float64 CPU oracle (test infrastructure only; see vmla_oracle.py)."""
