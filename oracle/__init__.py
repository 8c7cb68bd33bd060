"""Float64 CPU oracle for the JoLT / FlashJoLT compress, allocate and decompress path.

TEST INFRASTRUCTURE ONLY.  This package is the slow, plain, obviously-correct
restatement of the method that the CUDA library is checked against.  Only the
test-suite, ``__graft_entry__.smoke()`` and ``bench.py``'s CPU-baseline /
reference arm may import it.  The library never calls it, and it shares no code
with the library: it implements its own random-number generator, rounding,
Hadamard transform, quantiser, byte accounting and allocation from the pages'
description.

Parity status of each function is stated in ``jolt_ref``'s module docstring.
"""
from .jolt_ref import *  # noqa: F401,F403
