"""Float64 CPU oracle for the HARP rotation (test infrastructure only)."""
