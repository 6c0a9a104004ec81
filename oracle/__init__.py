"""CPU oracle of the skew-aware MoE forward layer (test infrastructure only)."""
