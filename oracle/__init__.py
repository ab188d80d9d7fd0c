"""CPU oracle for the 8-bit quantized linear layer (test infrastructure only)."""
