"""B200-native QK-Norm and FlashNorm (placeholder; the binding lands with the C ABI)."""
