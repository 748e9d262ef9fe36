"""Plain CPU oracle for routed HGA attention (test infrastructure only; see oracle.py)."""
