"""Float64 CPU oracle of the hybrid-block decode step (test infrastructure only)."""
from .hs2_oracle import *  # noqa: F401,F403
