"""Float64 CPU oracle of the routed MoE FFN forward pass.

TEST INFRASTRUCTURE ONLY: imported by ``tests/``, ``__graft_entry__.smoke()``
and the CPU-baseline legs of ``bench.py``, never by the CUDA library.  It
shares no code with the library; see ``moe_oracle.py`` for what it computes
and which passage of the pages each step follows.
"""

from . import moe_oracle  # noqa: F401
from .moe_oracle import *  # noqa: F401,F403
