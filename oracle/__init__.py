"""Float64 CPU oracle (test infrastructure only; see logmel_oracle)."""
from .logmel_oracle import *  # noqa: F401,F403
