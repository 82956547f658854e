"""CPU oracle (test infrastructure only; see ternary_oracle's header)."""
from .ternary_oracle import *  # noqa: F401,F403
from . import ternary_oracle  # noqa: F401
