"""Float64 CPU oracle for ZHA (test infrastructure only; see oracle.py)."""
