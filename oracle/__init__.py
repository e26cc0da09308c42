"""fp64 CPU oracle of the MSA forward pass (test infrastructure only)."""
