"""CPU oracle for one FOCUS focused denoising step -- TEST INFRASTRUCTURE ONLY.

Only `tests/`, `__graft_entry__.smoke()` and the CPU-baseline leg of `bench.py`
may import this package.  The product path (the CUDA library and its Python
binding) never calls it; it shares no code with that path.

Everything is float64 numpy, one request and one head at a time, in the order
the method states.  See `focus_oracle` for the step and its citations.

Parity pins: every function here is pinned by tests under `tests/` against
closed forms, invariants, brute force and an independently written dense
forward.  The one part with no such pin -- whether the importance delta really
predicts decodability -- is method quality, which needs trained weights and
datasets; for that "parity unpinned" holds (the oracle computes what the rule
says, nobody here can check that the rule works).
"""
from .focus_oracle import (  # noqa: F401
    OracleResult, focus_step, rms_norm, rope, attention, importance_from_probs,
    select_positions, compact_rows, lm_head_conf, threshold_decode, silu,
)
