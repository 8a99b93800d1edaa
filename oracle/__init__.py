"""CPU oracle of the int4 routed-expert MoE step -- TEST INFRASTRUCTURE.

Only ``tests/``, ``__graft_entry__.smoke()`` and ``bench.py``'s CPU-baseline
and reference legs may import this package (``__graft_entry__.build()``
compiles its C part).  It shares no code with the CUDA library.

Two statements of the same layer: ``oracle/moe.py`` (numpy, float64) and
``oracle/c/moe_ref.c`` (plain C, double; loaded by ``oracle/cref.py``).  Every
function of each is pinned (``tests/test_oracle_pins.py``,
``tests/test_oracle_c.py``), each set of pins is mutation-tested, and the two
are checked against each other on seeded layers.
"""
from .moe import *  # noqa: F401,F403
