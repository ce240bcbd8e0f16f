"""fp64 CPU oracle for piecewise sparse attention — test infrastructure only (see pisa_oracle)."""
