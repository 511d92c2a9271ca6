"""CPU oracle for the rotated W4A4 linear layer (test infrastructure only)."""
