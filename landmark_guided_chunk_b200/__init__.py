"""B200-native Hierarchical Sparse Attention (HSA) forward path (placeholder; the binding lands with the C-ABI)."""
