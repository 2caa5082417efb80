"""CPU oracle of the DSA hot path: test infrastructure only, never called by the library."""
