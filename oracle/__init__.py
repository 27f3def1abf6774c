"""fp64 CPU oracle for multi-scale retention -- test infrastructure only."""
