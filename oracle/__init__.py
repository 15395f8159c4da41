"""CPU float64 oracle for the R2L sidecar forward, the gradient of its scan and of a whole hook.

TEST INFRASTRUCTURE ONLY: imported by ``tests/``, by ``smoke()`` and by the
CPU-baseline legs of ``bench.py``; never by the library.
"""
from .r2l_oracle import *  # noqa: F401,F403
from .scan_backward import *  # noqa: F401,F403
from .sidecar_backward import *  # noqa: F401,F403
