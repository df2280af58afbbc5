"""fp64 CPU oracle for linear cross-entropy: test infrastructure, never called by the CUDA path."""
