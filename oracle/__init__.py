"""CPU oracle package (test infrastructure only; see csa_oracle's header)."""
