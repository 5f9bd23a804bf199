"""Float64 CPU oracle (test infrastructure only; see gqa_oracle)."""
from .gqa_oracle import *  # noqa: F401,F403
