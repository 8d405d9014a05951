"""CPU oracle (test infrastructure only; see exactmoe_oracle)."""
