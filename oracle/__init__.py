"""CPU oracle (test infrastructure only).

Only the tests, the smoke check and the CPU-baseline leg of the benchmark may
import this package.  The CUDA library never imports, links or calls it.
"""
from .bitlinear_oracle import *  # noqa: F401,F403
from . import bitlinear_oracle as core  # noqa: F401
