"""fp64 CPU oracle of the sparse MoE FFN layer forward.

Test infrastructure: only tests/, __graft_entry__.smoke() and bench.py's
CPU-baseline leg may import it.  It shares no code with the CUDA library.
"""
from .moe_oracle import *  # noqa: F401,F403
