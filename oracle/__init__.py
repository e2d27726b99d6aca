"""fp64 CPU oracle for MLA latent-KV decode (test infrastructure only; see mla_oracle.py)."""
from .mla_oracle import *  # noqa: F401,F403
from .mla_oracle import ROPE_BASE  # noqa: F401
