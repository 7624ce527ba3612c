"""CPU oracle for the MiniMax H3 DiT block hot path.

TEST INFRASTRUCTURE ONLY.  Only the test suite, ``__graft_entry__.smoke()``
and the benchmark's CPU-baseline / reference arm may import or run this
package.  The product path (the ``h3b`` C ABI and its Python binding) never
imports it and shares no code with it.

Everything here is plain numpy: fp64 for floating point, int64 for the integer
GEMM, fp32 exactly where the quantisation rule fixes fp32.  Each function
states the definition it writes out and where it comes from.  Parity status of
every function is listed in ``oracle.dit.PINS``.
"""
from .dit import *  # noqa: F401,F403
