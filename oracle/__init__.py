"""CPU oracle (test infrastructure only; see saf3r_oracle)."""
from .saf3r_oracle import *  # noqa: F401,F403
