"""Float64 CPU oracle (test infrastructure only; the library never imports it)."""
from .fva_oracle import *  # noqa: F401,F403
from . import rlb_oracle  # noqa: F401
from . import sasa_oracle  # noqa: F401
