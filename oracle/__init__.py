"""CPU oracle of the int4 routed-expert MoE step -- TEST INFRASTRUCTURE.

Only ``tests/``, ``__graft_entry__.smoke()`` and ``bench.py``'s CPU-baseline
and reference legs may import this package.  It shares no code with the CUDA
library; see ``oracle/moe.py`` for what it computes and which passages it
follows.  Every function is pinned by ``tests/test_oracle_pins.py``.
"""
from .moe import *  # noqa: F401,F403
