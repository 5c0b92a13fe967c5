"""CPU oracle (test infrastructure only; see muon_oracle's header)."""
from .muon_oracle import *  # noqa: F401,F403
