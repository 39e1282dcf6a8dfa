"""fp64 CPU oracle of the MoE-layer forward. Test infrastructure only: the
CUDA library never imports it."""
from .moe_oracle import *  # noqa: F401,F403
