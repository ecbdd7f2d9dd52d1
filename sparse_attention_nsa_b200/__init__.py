"""B200-native Native Sparse Attention (placeholder until the binding lands)."""
