"""FP64 CPU oracle of the Muse Spark Open latent-MoE block (test infrastructure only).

This package is the slow, obviously-correct definition that the CUDA path is checked
against: latent_moe.py and nvfp4.py in numpy (every mode, used by the parity tests), and
latent_moe_ref.c, the same block definition as a plain C program in double precision
(loaded through cref.py; pinned and compared with the numpy version in the tests). Only
tests/, __graft_entry__.smoke() and bench.py's cpu_baseline / reference leg may import it.
It shares no code with the CUDA library and never imports it.
"""
from .latent_moe import *  # noqa: F401,F403
from .nvfp4 import *  # noqa: F401,F403
