"""fp64 CPU attention oracle -- test infrastructure only (see oracle.py)."""
