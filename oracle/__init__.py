"""CPU oracle (test infrastructure only; see lens_oracle's header)."""
