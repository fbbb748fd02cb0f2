"""CPU oracle for the ARCHead packed LM-head path.  TEST INFRASTRUCTURE ONLY.

Only tests, the smoke check and the benchmark's CPU-baseline leg import this package.
The GPU library does not import, link or call it, and it imports nothing from the GPU
library.
"""
from .archead_oracle import *  # noqa: F401,F403
