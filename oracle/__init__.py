"""CPU float64 oracle of the RTPurbo decode step (test infrastructure; see rtp_oracle)."""
from .rtp_oracle import *  # noqa: F401,F403
