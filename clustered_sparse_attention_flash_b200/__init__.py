"""B200-native SVG-EAR sparse attention.

The operator runs entirely in libsvgear.so (hand-written CUDA for sm_100a,
C ABI in include/svgear.h); `svgear` is its ctypes binding and `synth` the
seeded synthetic-input generator.
"""
from . import svgear, synth  # noqa: F401

__all__ = ["synth", "svgear"]
