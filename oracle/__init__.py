"""CPU fp64 oracle of the top-k routed MoE FFN forward pass.

TEST INFRASTRUCTURE ONLY. Only `tests/`, `__graft_entry__.smoke()` and the
CPU-baseline leg of `bench.py` may import this package. The product path (the
CUDA library and its Python binding) never imports, links or runs it, and it
shares no code with that path.
"""
from .moe_oracle import *  # noqa: F401,F403
