"""CPU oracle (test infrastructure only; see ``minf_oracle``)."""
