"""CPU oracle for the SVG-EAR operator (test infrastructure only)."""
from .svgear_oracle import *  # noqa: F401,F403
