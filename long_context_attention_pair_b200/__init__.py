"""B200-native per-RoPE-wavelength windowed attention (binding is added with the C-ABI library)."""
