"""fp64 CPU oracle (test infrastructure only; see prox_oracle's header)."""

from .prox_oracle import *  # noqa: F401,F403
from . import prox_oracle  # noqa: F401
