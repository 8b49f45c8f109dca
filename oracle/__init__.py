"""CPU oracle of the MoE expert layer (test infrastructure; never on the product path)."""
