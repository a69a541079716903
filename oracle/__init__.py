"""CPU oracle (test infrastructure only; see i8q_oracle's module docstring)."""
from .i8q_oracle import *  # noqa: F401,F403
