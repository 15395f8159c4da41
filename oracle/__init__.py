"""CPU float64 oracle for the R2L sidecar forward and the gradient of its scan.

TEST INFRASTRUCTURE ONLY: imported by ``tests/``, by ``smoke()`` and by the
CPU-baseline legs of ``bench.py``; never by the library.
"""
from .r2l_oracle import *  # noqa: F401,F403
from .scan_backward import *  # noqa: F401,F403
