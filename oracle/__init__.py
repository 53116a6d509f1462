"""CPU oracle (test infrastructure only; see dlm_oracle.py's header)."""
from .dlm_oracle import *  # noqa: F401,F403
