"""Writes prefix_losses_<config>.json: oracle per-token losses of a prefix of
a full-size workload, for the full-size GPU parity tests.

By causality (算法 1 of the reading notes scores every position of a chunk
before that chunk's targets update W), the losses of positions 0 .. T'-2 of
a T'-token run equal those of the full T-token run.  The oracle cannot run a
whole 128K-token prefill in a test, so it runs T' tokens here, once, and the
GPU test compares the positions stored below with its own full-length run.

  2.7b: T' = 1536, one full chunk with its SGD update and half of the next;
  760m: T' = 17920, which crosses the 16 384-position boundary where the
        GPU path starts its second super-chunk of fast-weight-free blocks
        (second bottom-ring pass, RoPE table rebase, windows straddling the
        boundary).  Stored: positions 0 .. 1534 and 15 360 .. 17 918.

Every value comes from oracle.prefill on the seeded inputs of synth/; nothing
here reads the CUDA library.

Run: python tests/golden/make_prefix_losses.py [2.7b] [760m]
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

HERE = os.path.dirname(os.path.abspath(__file__))

# config -> (prefix length T', stored position ranges [a, b))
PLANS = {
    "2.7b": (1536, [(0, 1535)]),
    "760m": (17920, [(0, 1535), (15360, 17919)]),
}


def path_for(name):
    return os.path.join(HERE, f"prefix_losses_{name}.json")


def make(name):
    T1, ranges = PLANS[name]
    cfg = synth.get_config(name)
    w = synth.make_weights(cfg, keep_bits=False)
    toks = synth.tokens(cfg)
    t0 = time.time()
    res = oracle.prefill(oracle.Model(cfg, w.arrays), toks[:T1])
    out = {
        "config": name,
        "prefix_tokens": T1,
        "source": "oracle.prefill (fp64) on synth.tokens / synth.make_weights of this config; "
                  "losses of the listed positions of a T'-token run",
        "oracle_seconds": round(time.time() - t0, 1),
        "ranges": [list(r) for r in ranges],
        "losses": [[float(v) for v in res.losses[a:b]] for a, b in ranges],
        "chunk_mean": [float(m) for m in res.chunk_mean],
    }
    with open(path_for(name), "w") as fh:
        json.dump(out, fh)
    print(f"{name}: T'={T1} in {out['oracle_seconds']} s -> {path_for(name)}")


def load(name):
    """(ranges, list of float64 arrays) of a stored prefix."""
    with open(path_for(name)) as fh:
        js = json.load(fh)
    return [tuple(r) for r in js["ranges"]], [np.asarray(v, dtype=np.float64) for v in js["losses"]]


if __name__ == "__main__":
    for n in (sys.argv[1:] or list(PLANS)):
        make(n)
