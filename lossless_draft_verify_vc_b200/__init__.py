"""B200-native (sm_100a) hot path of VeriCache: draft attention over a
compressed KV cache, block verification attention over the full cache, and
greedy acceptance, behind the C ABI declared in include/vc.h.

``vc`` is the ctypes binding of that ABI; ``synth`` draws seeded synthetic
inputs; ``build`` compiles libvc_b200.so for sm_100a.
"""

from . import synth  # noqa: F401
from . import vc  # noqa: F401
