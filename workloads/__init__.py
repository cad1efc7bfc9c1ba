"""Seeded synthetic inputs shared by the tests and the benchmark.

This package only draws random numbers with fixed seeds and shapes; it holds
none of the BitLinear arithmetic, and neither the oracle nor the CUDA library
imports it.
"""

from .inputs import *  # noqa: F401,F403
