"""fp64 CPU oracle of one MoE layer's forward pass.

Test infrastructure only: ``tests/``, ``__graft_entry__.smoke()`` and the
CPU-baseline legs of ``bench.py`` may import it; the CUDA library never does.
"""
from .moe_oracle import *  # noqa: F401,F403
from .moe_oracle import __all__  # noqa: F401
