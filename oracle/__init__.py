"""fp64 CPU oracle (test infrastructure only; see hs2_oracle's header)."""
