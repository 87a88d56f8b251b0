"""CPU oracle for the streaming-experts MoE layer (test infrastructure).

Only the tests, ``__graft_entry__.smoke()`` and the benchmark's CPU baseline
import this package.  It wraps the plain C oracle (``moe_oracle.c``) with
numpy arrays; it never touches the CUDA library.
"""
from .oracle import *  # noqa: F401,F403
