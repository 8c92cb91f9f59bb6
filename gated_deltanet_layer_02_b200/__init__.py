"""B200-native Gated DeltaNet layer (placeholder; binding added with the C-ABI)."""
