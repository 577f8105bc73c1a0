"""CPU oracle (test infrastructure only; see nf4_oracle.py)."""
from .nf4_oracle import *  # noqa: F401,F403
