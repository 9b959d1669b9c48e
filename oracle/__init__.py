"""FP64 CPU oracle of the Muse Spark Open latent-MoE block (test infrastructure only).

This package is the slow, obviously-correct definition that the CUDA path is checked
against. Only tests/, __graft_entry__.smoke() and bench.py's cpu_baseline / reference
leg may import it. It shares no code with the CUDA library and never imports it.
"""
from .latent_moe import *  # noqa: F401,F403
from .nvfp4 import *  # noqa: F401,F403
