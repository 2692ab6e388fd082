"""float64 CPU oracle of the routed MoE FFN — TEST INFRASTRUCTURE.

Only ``tests/``, ``__graft_entry__.smoke()`` and ``bench.py``'s cpu_baseline and
``--impl reference`` legs may import anything here.  The product path (the
``quantised_expert_decode_b200`` package and its CUDA library) never does.
"""
from . import moe  # noqa: F401
