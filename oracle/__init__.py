"""CPU fp64 oracle (test infrastructure only; see xattn_oracle.py)."""
from .xattn_oracle import *  # noqa: F401,F403
from .xattn_oracle import __all__  # noqa: F401
