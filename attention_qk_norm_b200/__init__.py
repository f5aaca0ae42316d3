"""QK-Norm for B200 (placeholder until the CUDA library lands)."""
