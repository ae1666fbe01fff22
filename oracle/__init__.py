"""fp64 CPU oracle for Wall Attention (test infrastructure only; see wall_oracle.py)."""
