"""B200-native AB-Attention hot path (placeholder: binding added with the library)."""
