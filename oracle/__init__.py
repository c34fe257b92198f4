"""Float64 oracle of the routed MoE block.  Test infrastructure only: the
tests, the smoke check and the benchmark's CPU-baseline leg import it; the
CUDA path never does."""
from .moe_oracle import *  # noqa: F401,F403
