"""B200-native paged KV-cache decode path (placeholder; the binding follows)."""
