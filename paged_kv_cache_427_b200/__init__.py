"""B200-native paged KV-cache decode attention (placeholder; the binding lands with the library)."""
