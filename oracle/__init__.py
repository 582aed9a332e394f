"""Float64 CPU oracle for the DiT-block hot path (test infrastructure only)."""
