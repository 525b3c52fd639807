"""CPU oracle for Block-GTQ / TQ-MSE packed-KV decode attention.

TEST INFRASTRUCTURE ONLY. Nothing on the product path imports, calls or links this
package: only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` use it. It shares no code with ``packed_cache_decode_b200`` (the CUDA
library); the two meet only in the seeded input generator
``packed_cache_decode_b200.synth``, which holds none of the method's arithmetic.

Every function is plain numpy in float64 and follows the passage it cites. Parity
status of each function is listed in the header of ``bgtq_oracle``.
"""
from .bgtq_oracle import *  # noqa: F401,F403
