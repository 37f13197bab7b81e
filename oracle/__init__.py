"""CPU oracle (test infrastructure only; never part of the product path)."""
