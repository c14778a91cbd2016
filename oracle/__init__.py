"""CPU oracle for the MoE layer (test infrastructure; see moe_oracle.py)."""
