"""B200-native NVFP4 attention (placeholder; the binding is added with the C-ABI)."""
