"""fp64 CPU oracle of the hybrid compressed attention core (test infrastructure only)."""
from .dsv4_oracle import *  # noqa: F401,F403
