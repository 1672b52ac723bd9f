"""B200-native FMDQ differential linear (placeholder)."""
