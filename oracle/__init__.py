"""CPU oracle (test infrastructure only; see flexq_oracle)."""
