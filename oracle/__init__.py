"""fp64 CPU oracle for exact attention (test infrastructure only; never on the product path)."""
