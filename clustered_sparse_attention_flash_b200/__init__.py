"""B200-native SVG-EAR sparse attention (binding filled in with the CUDA library)."""
