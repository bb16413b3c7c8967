"""CPU oracle for LSH attention: test infrastructure, not part of the product path."""
