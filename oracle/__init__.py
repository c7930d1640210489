"""fp64 CPU oracle for Attention State Memory (test infrastructure only)."""
