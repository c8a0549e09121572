"""fp64 CPU oracle of SSA dual-stream attention (test infrastructure only)."""
