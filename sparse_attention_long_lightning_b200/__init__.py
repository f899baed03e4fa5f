"""B200-native SALA hybrid-attention hot path (placeholder; binding added with the library)."""
