"""CPU oracle package (test infrastructure only; see csffn_oracle's header)."""
from .csffn_oracle import *  # noqa: F401,F403
from .csffn_oracle import RMS_EPS  # noqa: F401
