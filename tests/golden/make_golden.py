"""Writes tests/golden/worked_example.json.

The inputs are a hand-made 4-token, 2-block example (P = N = 2) whose per-token
decay is exactly 1/2: dt = 1/2 and A = -2 ln 2, so a = exp(dt A) = 1/2.  The
stored output is the fp64 oracle's; the test recomputes the same example in
exact rational arithmetic and checks both.  This script calls only the oracle.
"""
import json
import math
import os
import sys

import numpy as np

HERE = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, os.path.dirname(os.path.dirname(HERE)))

import oracle  # noqa: E402

A = -2.0 * math.log(2.0)
EXAMPLE = {
    "about": ("Hand-made worked example of eq. (1) with the forward boundary state (eq. (10)), "
              "block-local reverse (eq. (12)) and the sum (eq. (13)) of 'Training Hybrid Block "
              "Diffusion Language Models with Partial Bidirectionality'; decay a = 1/2 per token."),
    "block_len": 2,
    "h0": [[1.0, -0.5], [0.25, 2.0]],
    "fwd": {"dt": [0.5, 0.5, 0.5, 0.5], "A": A, "D": 0.5,
            "x": [[1.0, -2.0], [0.5, 1.0], [-1.0, 0.0], [2.0, 1.5]],
            "B": [[1.0, 0.5], [-0.5, 2.0], [0.0, 1.0], [1.5, -1.0]],
            "C": [[2.0, -1.0], [0.5, 0.25], [-1.0, 1.0], [1.0, 2.0]]},
    "rev": {"dt": [0.5, 0.5, 0.5, 0.5], "A": A, "D": -1.5,
            "x": [[0.5, 1.0], [1.0, -1.0], [2.0, 0.5], [-0.5, -2.0]],
            "B": [[0.25, 1.0], [1.0, -1.0], [-2.0, 0.5], [0.5, 0.5]],
            "C": [[1.0, 1.0], [-1.0, 0.5], [0.25, -0.5], [2.0, 0.0]]},
}


def main():
    L = 4

    def as_dir(d):
        return {"x": np.array(d["x"]).reshape(1, L, 1, 2), "dt": np.array(d["dt"]).reshape(1, L, 1),
                "B": np.array(d["B"]).reshape(1, L, 1, 2), "C": np.array(d["C"]).reshape(1, L, 1, 2),
                "A": np.array([d["A"]]), "D": np.array([d["D"]])}

    shape = dict(batch=1, seqlen=L, nheads=1, headdim=2, dstate=2, ngroups=1, block_len=2)
    y, st, fin = oracle.prefix(shape, as_dir(EXAMPLE["fwd"]), as_dir(EXAMPLE["rev"]),
                               h0=np.array(EXAMPLE["h0"]).reshape(1, 1, 2, 2))
    out = dict(EXAMPLE)
    out["oracle_output"] = {"y": y.reshape(L, 2).tolist(), "states": st.reshape(2, 2, 2).tolist(),
                            "final_state": fin.reshape(2, 2).tolist()}
    with open(os.path.join(HERE, "worked_example.json"), "w") as f:
        json.dump(out, f, indent=1)


if __name__ == "__main__":
    main()
