"""fp64 CPU oracle of the FwPKM step (test infrastructure only)."""
