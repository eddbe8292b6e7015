"""CPU oracle for the SS1 layer forward (test infrastructure only; see ss1_oracle)."""

from .ss1_oracle import *  # noqa: F401,F403
from .ss1_oracle import __all__  # noqa: F401
