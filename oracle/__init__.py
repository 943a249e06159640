"""Float64 CPU oracle of the SuperGlue matcher (test infrastructure only)."""
from .superglue_oracle import *  # noqa: F401,F403
