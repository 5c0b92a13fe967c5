"""CPU oracle (test infrastructure only; see muon_oracle's header)."""
from .muon_oracle import *  # noqa: F401,F403
from .muon_oracle import bank_muon_step  # noqa: F401
