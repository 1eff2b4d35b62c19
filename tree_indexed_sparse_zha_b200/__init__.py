"""B200-native ZHA hot path (placeholder; the binding is filled in below)."""
