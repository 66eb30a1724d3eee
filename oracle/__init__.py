"""CPU float64 oracle of the affine autoregressive flow block (test infrastructure only)."""
