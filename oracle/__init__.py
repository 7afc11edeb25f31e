"""fp64 CPU oracle of the DP-GRAPE step (test infrastructure only; see grape_oracle)."""
from .grape_oracle import *  # noqa: F401,F403
from . import grape_oracle  # noqa: F401
