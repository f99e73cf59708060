"""Writes tests/golden/tiny_oracle_case.json by calling only the oracle.

The pages print no worked input/output example, so this fixture is a
regression record of the (pinned) oracle on one tiny seeded case: inputs are
bf16-representable values drawn by the shared seeded generator, outputs are the
oracle's fp64 results.  Re-run only when the oracle's arithmetic is changed on
purpose, and name the passage that justifies the change in the commit.
"""
import json
import math
import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
sys.path.insert(0, ROOT)

import oracle  # noqa: E402
from exact_attention_108_b200.workloads import make_inputs, to_f64  # noqa: E402


def main():
    B, H, N, d, seed = 1, 1, 16, 8, 7
    q, k, v, do = (to_f64(t) for t in make_inputs(B, H, N, d, seed))
    scale = 1.0 / math.sqrt(d)
    case = {"B": B, "H": H, "N": N, "d": d, "seed": seed, "scale": scale,
            "q": q.tolist(), "k": k.tolist(), "v": v.tolist(), "do": do.tolist()}
    for causal in (False, True):
        o, lse = oracle.ref_fwd(q, k, v, causal, scale)
        dq, dk, dv = oracle.ref_bwd(q, k, v, do, causal, scale)
        case["causal" if causal else "full"] = {
            "o": o.tolist(), "lse": lse.tolist(),
            "dq": dq.tolist(), "dk": dk.tolist(), "dv": dv.tolist()}
    out = os.path.join(os.path.dirname(os.path.abspath(__file__)), "tiny_oracle_case.json")
    with open(out, "w") as f:
        json.dump(case, f, indent=0)


if __name__ == "__main__":
    main()
