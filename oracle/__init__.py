"""fp64 CPU oracle (test infrastructure only; see ``seer_oracle``)."""
from .seer_oracle import *  # noqa: F401,F403
