"""CPU oracle (test infrastructure only; see jfa_oracle's module docstring)."""
from .jfa_oracle import *  # noqa: F401,F403
