"""fp64 CPU oracle of the DSpark round (test infrastructure only)."""
