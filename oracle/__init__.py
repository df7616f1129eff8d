"""Float64 CPU oracle (test infrastructure only; see mlra_oracle.py)."""
from .mlra_oracle import *  # noqa: F401,F403
