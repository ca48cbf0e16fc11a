"""fp64 CPU oracle for block-compressed attention (test infrastructure only)."""
