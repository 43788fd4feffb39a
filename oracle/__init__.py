"""fp64 CPU oracle for the routed MoE decode layer (test infrastructure).

Only the test suite, ``__graft_entry__.smoke()`` and the CPU-baseline /
reference arm of ``bench.py`` may import this package. It shares no code with
the CUDA path and imports nothing from it. See ``moe_oracle`` for the
definitions and the passages of the pages each one follows.
"""

from . import moe_oracle  # noqa: F401
from .moe_oracle import *  # noqa: F401,F403
