"""fp64 CPU oracle for exact attention -- TEST INFRASTRUCTURE.

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline / reference
leg of ``bench.py`` may import this package.  The CUDA product path never
imports, links or calls it, and it shares no code with that path.

Parity status: every function here is pinned by tests that do not restate its
formula (library softmax / logsumexp on tiny inputs, closed forms, invariants,
central finite differences); see ``tests/test_oracle_pins.py``.
"""
from .oracle import (  # noqa: F401
    build_oracle,
    oracle_threads,
    fwd_rows,
    prob_row,
    bwd_rows,
    dense_fwd,
    dense_bwd,
    online_fwd,
    decode_rows,
)
