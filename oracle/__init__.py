"""CPU oracle (test infrastructure only; see bsa_oracle's header)."""
from .bsa_oracle import *  # noqa: F401,F403
