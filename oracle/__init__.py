"""fp64 CPU oracle of the CSA/HCA hot path (test infrastructure only; see csa_oracle)."""
from .csa_oracle import *  # noqa: F401,F403
