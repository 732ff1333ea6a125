"""CPU oracle for the Stable LatentMoE layer forward pass.

TEST INFRASTRUCTURE ONLY.  Only the tests, ``__graft_entry__.smoke()`` and the
``cpu_baseline`` / ``--impl reference`` legs of ``bench.py`` may import it.
The CUDA library never imports, links or calls anything here, and nothing
here imports the CUDA library.

Two independent restatements of the method, with the same functions:
  * the fp64 C++ oracle (``moe_oracle.cpp``, std::thread workers), exported
    here and used by every parity check and by the CPU baseline;
  * a plain fp64 PyTorch-CPU restatement (``moe_oracle.py``, available as
    ``oracle.torch_ref``), kept as a cross-check of the C++ one.

Every function of both is pinned by CPU tests against something other than
itself (closed forms, invariants, brute force, published tables); see
``tests/test_oracle_pins.py``.  No function here is "parity unpinned".
"""
from . import moe_oracle as torch_ref  # noqa: F401
from .cpp_oracle import *  # noqa: F401,F403
from .cpp_oracle import __all__, num_threads  # noqa: F401
