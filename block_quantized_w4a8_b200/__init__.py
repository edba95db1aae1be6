"""Block-quantized W4A8 matmul for NVIDIA B200 (placeholder; the binding lands next)."""
