"""Writes tests/golden/oracle_regression.json: the fp64 oracle's results on one small seeded
layer (B = 2, L = 24, 4 query heads over 2 KV heads, d = 8, bf16 inputs, q = 6, tau = 0.05).
Scores, budget and index lists are stored in full (floats as exact hex); the attention rows
and the layer output as the SHA-256 of their fp64 bytes plus their first values.

The values come from `oracle/` alone (the seeded input generator supplies the inputs).  They
are not a statement of what the pages print: the pages give no worked example.  They pin
the oracle against unintended changes of its arithmetic; a deliberate change regenerates
this file, and its commit names the passage or reading that justifies it.

    python tests/golden/make_oracle_regression.py
"""
import json
import os
import sys

import numpy as np
import torch

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(os.path.dirname(HERE))
sys.path.insert(0, ROOT)

CASE = dict(B=2, L=24, H=4, Hkv=2, d=8, seed=11, q=6, tau=0.05)


def compute():
    import oracle
    from token_sparse_attention_dtc_b200.inputs import make_inputs

    c = CASE
    x = make_inputs(c["B"], c["L"], c["H"], c["Hkv"], c["d"], torch.bfloat16, seed=c["seed"])
    r = oracle.layer(x["Q"], x["K"], x["V"], x["X"], c["q"], c["tau"])
    return digest(r)


def digest(r):
    import hashlib

    f64 = lambda a: np.ascontiguousarray(np.asarray(a, np.float64))
    hexes = lambda a: [float(v).hex() for v in f64(a).ravel()]
    big = lambda a: dict(sha256=hashlib.sha256(f64(a).tobytes()).hexdigest(),
                         shape=list(f64(a).shape), first=hexes(f64(a).ravel()[:16]))
    return dict(
        case=CASE,
        s_h=hexes(r["s_h"]), s_l=hexes(r["s_l"]),
        Lkeep=[int(v) for v in np.asarray(r["Lkeep"]).ravel()],
        idx=[int(v) for v in np.asarray(r["idx"]).ravel()],
        Oh=big(r["Oh"]), Y=big(r["Y"]))


if __name__ == "__main__":
    out = os.path.join(HERE, "oracle_regression.json")
    with open(out, "w") as f:
        json.dump(compute(), f, indent=0)
        f.write("\n")
    print("wrote", out)
