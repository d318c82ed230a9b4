"""Plain, slow CPU oracle of the DraftAttention2 hot path -- TEST INFRASTRUCTURE ONLY.

Only `tests/`, `__graft_entry__.smoke()` and the `cpu_baseline` / reference leg of
`bench.py` may import this package. The CUDA library never calls it, and the two share
no code: the oracle is written from the method's description in numpy (fp64 unless a
step is defined in fp32), the CUDA path from its own design.
"""
from .da2_oracle import *  # noqa: F401,F403
