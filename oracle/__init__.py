"""CPU oracle (test infrastructure only; see w4_oracle's header)."""
from .w4_oracle import *  # noqa: F401,F403
