"""fp64 CPU oracle of the MoE FFN layer: test infrastructure only (see moe_oracle)."""
