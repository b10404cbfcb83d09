"""B200-native chunkwise gated delta rule (placeholder; binding added with the C-ABI)."""
