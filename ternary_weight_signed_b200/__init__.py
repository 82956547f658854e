"""B200-native ternary-g128 linear layer with a signed block-Hadamard rotation.

The compute path lives in ``libternary_b200.so`` (hand-written CUDA for
sm_100a behind a C ABI, declared in ``include/ternary_b200.h``).  The Python
names mirror the C entry points and only marshal arguments; importing this
package does not load the library, calling a binding does, and a missing
library raises instead of falling back to anything else.
"""
from . import inputs  # noqa: F401  (seeded generators, no layer arithmetic)

__all__ = ["inputs"]
