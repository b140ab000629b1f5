"""CPU oracle for the routed MoE layer (test infrastructure only; see oracle.py)."""
