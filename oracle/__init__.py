"""CPU oracle (test infrastructure).  See w4a4_oracle.py."""
from .w4a4_oracle import *  # noqa: F401,F403
from . import w4a4_oracle as core  # noqa: F401
