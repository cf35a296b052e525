"""Float64 CPU oracle (test infrastructure only; see paro_ref)."""
