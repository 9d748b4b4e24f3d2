"""Float64 CPU oracle (test infrastructure only; see mao_oracle.py's header)."""
from .mao_oracle import *  # noqa: F401,F403
