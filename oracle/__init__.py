"""fp64 CPU oracle of the latent-KV chunk attention path (test infrastructure only)."""
from .vmla_oracle import *  # noqa: F401,F403
