"""fp64 CPU oracle (test infrastructure; see lrkv_oracle)."""
from .lrkv_oracle import *  # noqa: F401,F403
