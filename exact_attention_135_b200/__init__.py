"""B200-native fused exact attention (placeholder: the binding lands with the C library)."""
