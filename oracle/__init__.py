"""CPU oracle for the AWQ W4A16 path: test infrastructure only (see awq_oracle)."""
from .awq_oracle import *  # noqa: F401,F403
