"""CPU fp64 oracle (test infrastructure only; see paro_oracle.py)."""
from .paro_oracle import *  # noqa: F401,F403
