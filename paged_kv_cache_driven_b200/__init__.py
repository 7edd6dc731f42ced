"""B200-native paged KV cache decode path (placeholder; binding added with the boundary)."""
