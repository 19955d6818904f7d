"""CPU oracle (test infrastructure only).

Only ``tests/``, ``__graft_entry__.smoke()`` and ``bench.py``'s CPU-baseline
and reference legs may import this package. It shares no code with the CUDA
path in ``moe_routed_expert_top_b200``.
"""
from . import moe_oracle  # noqa: F401
