"""fp64 CPU oracle (test infrastructure only; see lmh_oracle's docstring for who may import it)."""
from .lmh_oracle import *  # noqa: F401,F403
from . import lmh_oracle  # noqa: F401
