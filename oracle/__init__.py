"""fp64 CPU oracle (test infrastructure only; see dsv4_oracle's header)."""
from .dsv4_oracle import *  # noqa: F401,F403
from . import dsv4_oracle  # noqa: F401
