"""CPU float64 oracle for the StateKV step (test infrastructure only)."""
