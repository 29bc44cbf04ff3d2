"""f64 CPU oracle (test infrastructure only; see kld_oracle.py)."""
from .kld_oracle import *  # noqa: F401,F403
from .kld_oracle import Q_FLOOR  # noqa: F401
