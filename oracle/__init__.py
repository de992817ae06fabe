"""CPU oracle (test infrastructure only): see vq_oracle."""
from .vq_oracle import *  # noqa: F401,F403
