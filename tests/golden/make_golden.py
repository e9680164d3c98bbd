"""Write tests/golden/oracle_small_cases.json from the oracle alone.

Run from the repository root:  python tests/golden/make_golden.py
The inputs come from the seeded generator; every expected value is computed by
the fp64 oracle (C build) and nothing else.
"""
import json
import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
sys.path.insert(0, ROOT)

import oracle  # noqa: E402
from exact_io_aware_93_b200.inputs import make_inputs  # noqa: E402

CASES = [
    dict(name="n16_d8_noncausal", N=16, d=8, seed=501, causal=False),
    dict(name="n16_d8_causal", N=16, d=8, seed=502, causal=True),
    dict(name="n9_d4_causal", N=9, d=4, seed=503, causal=True),
]


def main():
    out = []
    for c in CASES:
        t = make_inputs(1, 1, c["N"], c["d"], c["seed"], with_do=True)
        q, k, v, do = (t[n][0, :, 0].double().numpy() for n in ("q", "k", "v", "do"))
        scale = 1.0 / c["d"] ** 0.5
        o, lse = oracle.fwd_rows(q, k, v, scale, c["causal"])
        dq, _, dk, dv = oracle.bwd_rows(q, k, v, do, scale, c["causal"])
        out.append(dict(c, scale=scale, o=o.tolist(), lse=lse.tolist(), dq=dq.tolist(),
                        dk=dk.tolist(), dv=dv.tolist()))
    path = os.path.join(os.path.dirname(os.path.abspath(__file__)), "oracle_small_cases.json")
    with open(path, "w") as f:
        json.dump({"generator": "tests/golden/make_golden.py (oracle only)", "cases": out}, f,
                  indent=1)
        f.write("\n")


if __name__ == "__main__":
    main()
