"""Independent float64 CPU oracle (test infrastructure only; never imported by the library)."""
from . import wush_oracle  # noqa: F401
from .wush_oracle import *  # noqa: F401,F403
