"""fp64 CPU oracle of the quantized linear layer (test infrastructure only)."""
