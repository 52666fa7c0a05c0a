"""CPU oracle of the ZHA hot path (test infrastructure only; see zha_oracle)."""
