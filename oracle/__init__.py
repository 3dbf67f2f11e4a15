"""CPU float64 oracle (test infrastructure only; see bfmoe_oracle)."""
from .bfmoe_oracle import *  # noqa: F401,F403
