"""B200-native exact attention forward (placeholder; binding added with the kernel)."""
