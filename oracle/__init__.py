"""fp64 CPU oracle (test infrastructure only; see ``lcsa_oracle``)."""
from .lcsa_oracle import *  # noqa: F401,F403
from . import lcsa_oracle  # noqa: F401
