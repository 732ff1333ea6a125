"""CPU oracle for the Stable LatentMoE layer forward pass.

TEST INFRASTRUCTURE ONLY.  Only the tests, ``__graft_entry__.smoke()`` and the
``cpu_baseline`` / ``--impl reference`` legs of ``bench.py`` may import it.
The CUDA library never imports, links or calls anything here, and nothing
here imports the CUDA library: the oracle is an independent restatement of
the method in plain fp64 PyTorch CPU operations.

Every function is pinned by a CPU test against something other than itself
(closed forms, invariants, brute force, published tables); see
``tests/test_oracle_pins.py``.  No function here is "parity unpinned".
"""
from .moe_oracle import *  # noqa: F401,F403
from .moe_oracle import __all__  # noqa: F401
