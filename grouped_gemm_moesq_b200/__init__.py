"""paired-4:8 NVFP4 grouped sparse GEMM for routed MoE experts on B200."""
from .binding import *  # noqa: F401,F403
