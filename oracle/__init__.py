"""fp64 CPU oracle (test infrastructure only; see qmoe_oracle's header)."""
from .qmoe_oracle import *  # noqa: F401,F403
