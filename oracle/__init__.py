"""CPU fp64 oracle (test infrastructure only; never used by the product path)."""
from .vdn_oracle import *  # noqa: F401,F403
