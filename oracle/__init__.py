"""Float64 CPU oracle (test infrastructure; never imported by the CUDA path)."""
from .samba_oracle import *  # noqa: F401,F403
