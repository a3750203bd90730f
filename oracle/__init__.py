"""CPU oracle for the fused top-k Mixture-of-Experts layer.

TEST INFRASTRUCTURE ONLY.  Nothing in the product path may import, call or
execute this package: it is used by ``tests/``, by ``__graft_entry__.smoke()``
and by the ``cpu_baseline`` / ``--impl reference`` legs of ``bench.py``, and
by nothing else.  It shares no code with the CUDA library in
``moe_layer_top_b200/csrc``.
"""

from .moe_oracle import *  # noqa: F401,F403
