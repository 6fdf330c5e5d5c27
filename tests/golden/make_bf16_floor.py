"""Writes bf16_floor_<config>.json: the bf16 storage noise floor of the
per-token losses of the first chunk of a bf16 workload.

oracle/bf16_floor.py runs the oracle's fp64 forward twice on the seeded
inputs of synth/: exactly, and with every tensor the bf16 pipeline stores
as bf16 rounded there (attention and MLP norm outputs, q/k/v, q/k after
QK-norm and RoPE, attention probabilities, attention output, SwiGLU
activations, final norm output).  The per-position difference of the two
runs' losses is stored for positions 0 .. b-2 (the first chunk, scored
before any update), with its quantiles.  Nothing here reads the CUDA
library.

Run: python tests/golden/make_bf16_floor.py [2.7b] [125m] [760m]
"""
import json
import os
import sys
import time

ROOT = os.path.dirname(os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
sys.path.insert(0, ROOT)
import numpy as np  # noqa: E402

import oracle  # noqa: E402
import synth  # noqa: E402
from oracle import bf16_floor  # noqa: E402

HERE = os.path.dirname(os.path.abspath(__file__))


def make(name):
    cfg = synth.get_config(name)
    w = synth.make_weights(cfg, keep_bits=False)
    toks = synth.tokens(cfg)
    n = cfg.b - 1
    t0 = time.time()
    d = bf16_floor.floor(oracle.Model(cfg, w.arrays), toks, n)
    out = {
        "config": name,
        "positions": n,
        "source": "oracle.bf16_floor.floor: |loss(bf16 storage roundings) - loss(exact)|, fp64, W_init, "
                  "positions 0 .. b-2 of synth.tokens with synth.make_weights",
        "seconds": round(time.time() - t0, 1),
        "quantiles": {q: float(np.percentile(d, float(q))) for q in ("50", "90", "99", "99.5", "100")},
        "mean": float(d.mean()),
        "abs_err": [float(v) for v in d],
    }
    with open(os.path.join(HERE, f"bf16_floor_{name}.json"), "w") as fh:
        json.dump(out, fh)
    print(name, {k: round(v, 4) for k, v in out["quantiles"].items()}, "mean", round(out["mean"], 4),
          f"{out['seconds']} s")


if __name__ == "__main__":
    for n in (sys.argv[1:] or ["2.7b"]):
        make(n)
