"""Seeded synthetic inputs shared by the tests, the benchmark and the oracle's checks.

This package draws random numbers and shapes only. It holds none of the paged
attention arithmetic: no block counts, no slot addresses, no attention. Both the
CUDA path and the CPU oracle receive its outputs as plain inputs.
"""

from . import configs, synth  # noqa: F401
from .synth import *  # noqa: F401,F403
