"""B200-native pure W4A4 group-quantized GEMM (placeholder; the binding lands next)."""
