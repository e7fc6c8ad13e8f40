"""Plain fp64 CPU oracle of the DeepSeekMoE layer forward.

TEST INFRASTRUCTURE ONLY: the tests, the smoke check and the bench's CPU
baseline leg are the only callers.  Nothing here is shared with, or called by,
the CUDA product path.  See moe_oracle.py (bf16/fp32 layer) and fp8.py (E4M3
fine-grained quantisation and the emulating FP8 layer).

Parity pins: every function is pinned by the `-m "not gpu"` tests in
tests/test_oracle_pins.py against closed forms, brute force and values the
pages print.  The expert FFN numerics beyond the closed-form and hand-worked
cases are pinned only through those cases (partial pin, stated in the design
notes).
"""
from . import fp8, moe_oracle  # noqa: F401
