"""fp64 CPU oracle for the spatial/temporal sparse-attention path (test infrastructure)."""
from .svg_oracle import *  # noqa: F401,F403
