"""fp64 CPU oracle: test infrastructure only (see vsa_oracle's header)."""
