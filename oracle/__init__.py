"""fp64 CPU oracle of the gated delta-rule layer (test infrastructure only)."""
