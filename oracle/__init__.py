"""fp64 CPU oracle for exact masked softmax attention (test infrastructure only)."""
