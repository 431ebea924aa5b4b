"""CPU oracle for parity tests (test infrastructure; not part of the product path)."""
