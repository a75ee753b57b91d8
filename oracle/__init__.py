"""CPU oracle (test infrastructure only; see ress_oracle.py)."""
from .ress_oracle import *  # noqa: F401,F403
