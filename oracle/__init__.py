"""Double-precision CPU oracle for the LCA decode step (test infrastructure only)."""
