"""fp64 CPU oracle (test infrastructure only; see tqp_oracle's module docstring)."""
from .tqp_oracle import *  # noqa: F401,F403
from . import tqp_oracle  # noqa: F401
