"""CPU oracle for the MoE layer forward (test infrastructure, not product).

Only ``tests/``, ``__graft_entry__.smoke()`` and ``bench.py``'s CPU-baseline /
reference leg may import anything from here.  The CUDA library never calls it
and shares no code with it.
"""
from .moe_oracle import *  # noqa: F401,F403
from .moe_oracle import __all__  # noqa: F401
