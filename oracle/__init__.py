"""fp64 CPU oracle of the ISPA hot path (test infrastructure; see ispa_oracle)."""
from .ispa_oracle import *  # noqa: F401,F403
