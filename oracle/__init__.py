"""CPU oracle for the KnapSpec DP (test infrastructure only; see ks_oracle)."""
