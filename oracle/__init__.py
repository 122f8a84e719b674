"""CPU fp64 oracle (test infrastructure only; see starkv_oracle)."""
