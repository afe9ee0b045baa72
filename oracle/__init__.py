"""CPU oracle (test infrastructure only; see jetfire_oracle's header)."""
from .jetfire_oracle import *  # noqa: F401,F403
