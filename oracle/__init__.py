"""Float64 CPU oracle (test infrastructure only; see wsvd_oracle's header)."""
from .wsvd_oracle import *  # noqa: F401,F403
