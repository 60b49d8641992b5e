"""Writes tests/golden/tiny_seed0.json: the oracle's routing and output for the
first two tokens of the tiny configuration (hidden 512, intermediate 128,
32 routed experts + 1 shared, top-4, 4-bit, seed 0).  Calls only the oracle
(and, through it, the seeded input generator)."""
import json
import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402

import oracle  # noqa: E402
import fmoe_synth as synth  # noqa: E402


def main():
    shape = synth.CONFIGS["tiny"]["shape"]
    lay = oracle.synthetic_layer(0, 0, shape)
    out = {"config": "tiny", "seed": 0, "tokens": []}
    for t in range(2):
        x = oracle.bf16_to_f64(synth.gen_x_token(0, t, shape.hidden))
        r = lay.forward(x)
        out["tokens"].append({
            "token": t,
            "idx": [int(i) for i in r.idx],
            "w": [float(v) for v in r.w],
            "sigma": float(r.sigma),
            "y": [float(v) for v in r.y],
        })
    path = os.path.join(os.path.dirname(os.path.abspath(__file__)), "tiny_seed0.json")
    with open(path, "w") as f:
        json.dump(out, f)
    print(path)


if __name__ == "__main__":
    main()
