"""CPU float64 oracle of the WISE attention hot path (test infrastructure only)."""
