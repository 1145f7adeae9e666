"""Write ``oracle_snapshot.json``: oracle outputs for two small seeded cases.

Calls only the CPU oracle (and the seeded input generators).  The snapshot
guards the oracle's arithmetic against accidental change; a deliberate change
regenerates it, with the passage that justifies it named in the commit.

    python tests/golden/make_snapshot.py
"""
import json
import os
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, os.path.dirname(os.path.dirname(HERE)))

import oracle  # noqa: E402
from workloads import Spec, make_inputs  # noqa: E402

CASES = [Spec("snap_f32", 1, 2, 11, 8, 4, "f32", 101),
         Spec("snap_bf16", 2, 1, 9, 8, 3, "bf16", 102, qk_dist="laplace_negrows", v_sigma=2.0)]


def main():
    out = {"_about": "oracle (recurrence route) outputs and final states for small seeded "
                     "cases; written by make_snapshot.py from oracle/ only", "cases": []}
    for spec in CASES:
        inp = make_inputs(spec, threads=1)
        o, st, _ = oracle.recurrence(inp.q, inp.k, inp.v, inp.rope_cos, inp.rope_sin,
                                     spec.block_len, spec.eps)
        out["cases"].append({"spec": {f: getattr(spec, f) for f in spec.__dataclass_fields__},
                             "out": o.ravel().tolist(), "state": st.ravel().tolist()})
    with open(os.path.join(HERE, "oracle_snapshot.json"), "w") as f:
        json.dump(out, f, indent=0)


if __name__ == "__main__":
    main()
