"""fp64 CPU oracle for the GDN layer (test infrastructure only; see oracle.py)."""
