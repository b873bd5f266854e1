"""B200-native paged KV-cache attention (placeholder during bring-up)."""
