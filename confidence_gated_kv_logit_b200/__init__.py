"""B200-native CONF-KV decode-step hot path (placeholder during bring-up)."""
