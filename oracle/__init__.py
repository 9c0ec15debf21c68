"""Float64 CPU oracle for exact attention -- TEST INFRASTRUCTURE ONLY.

Only tests, the smoke check and the benchmark's CPU-baseline leg may import
this package.  The CUDA library never does, and this package never imports the
library.
"""
from .attention import *  # noqa: F401,F403
