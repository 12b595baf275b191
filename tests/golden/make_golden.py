"""Write oracle_small.json: a tiny seeded problem and the float64 oracle's outputs.
Calls only oracle/ (plus numpy's generator for the inputs)."""
import json
import os
import sys

import numpy as np

HERE = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, os.path.dirname(os.path.dirname(HERE)))
from oracle import rope_attn_ref as ref  # noqa: E402


def main():
    rng = np.random.default_rng(2024)
    shape = (1, 2, 6, 4)
    q, k, v, e = (np.round(rng.standard_normal(shape), 3) for _ in range(4))
    alpha = np.round(0.5 * rng.standard_normal(2), 3)
    out = {"shape": shape, "base": 10.0, "causal": True,
           "q": q.tolist(), "k": k.tolist(), "v": v.tolist(), "e": e.tolist(),
           "alpha": alpha.tolist()}
    r = ref.forward_backward(q, k, v, e, alpha, 10.0, True)
    for key in ("o", "lse", "dq", "dk", "dv", "dalpha"):
        out[key] = np.asarray(r[key]).tolist()
    out["L"] = r["L"]
    with open(os.path.join(HERE, "oracle_small.json"), "w") as f:
        json.dump(out, f, indent=1)


if __name__ == "__main__":
    main()
