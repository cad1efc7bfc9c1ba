"""CPU oracle for the BitNet b1.58 BitLinear training hot path.

TEST INFRASTRUCTURE ONLY. Only the test suite, the smoke check in
``__graft_entry__`` and the CPU-baseline leg of ``bench.py`` may import this
package. The CUDA library never calls it and shares no code with it.
"""

from .bitlinear_ref import *  # noqa: F401,F403
