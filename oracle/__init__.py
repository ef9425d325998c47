"""CPU oracle (test infrastructure only; see svg_oracle's header)."""
from .svg_oracle import *  # noqa: F401,F403
