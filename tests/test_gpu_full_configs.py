"""Parity at the full workload sizes, in the launch configuration bench.py
times (one sequence of T tokens through ttt_prefill).

The oracle cannot run a whole 128K-token prefill in a test, so it runs a
prefix: by causality (算法 1 of the reading notes scores every position of a
chunk before that chunk's targets update W), the losses of positions
0 .. T'-2 of the full GPU run equal those of a T'-token run.  T' covers one
full chunk (so an SGD update happens) and part of the next (scored with the
updated weights).  Where tests/golden/make_prefix_losses.py (oracle only)
stored a workload's prefix losses (2.7B; 760M, whose stored prefix crosses
the 16 384-position boundary where the GPU path starts the second
super-chunk of its fast-weight-free blocks) the test reads them; otherwise
(125M) the oracle runs the 1 536-token prefix here.  At full size the
2.7B run is also checked for properties that hold at any size: run-to-run
bit-identical losses, causality under a perturbed late token, finiteness.

Tolerances (bf16): every chunk's mean loss within 1e-2 absolute, and the
per-token loss within 5e-2 absolute at every compared position — unless the
bf16 storage floor of the workload itself exceeds 5e-2.  The floor is the
loss difference between the oracle's fp64 forward with and without the
bf16 roundings of the stored activations (oracle/bf16_floor.py, stored for
2.7B's first chunk in tests/golden/bf16_floor_2.7b.json); no bf16 pipeline
with these storage points can beat it.  Where it reaches past 5e-2 (2.7B),
the GPU's per-token errors must stay within the floor's distribution: the
50th, 90th and 99th percentiles and the maximum at most 1.25 times the
floor's, in each chunk compared."""
import json
import os

import numpy as np
import pytest
import torch

import oracle
import synth

from ._gpu_helpers import chunk_means

pytestmark = pytest.mark.gpu

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def _gpu_run(cfg, toks, weights_dev, ctx_cache):
    from test_long_context_b200.context import Context
    if "ctx" not in ctx_cache:
        ctx_cache["ctx"] = Context(cfg, weights_dev)
    ctx = ctx_cache["ctx"]
    ctx.reset()
    losses, _ = ctx.prefill(torch.from_numpy(np.asarray(toks, dtype=np.int32)).cuda())
    return losses.cpu().numpy().astype(np.float64)


def _stored_prefix(name):
    with open(os.path.join(GOLDEN, f"prefix_losses_{name}.json")) as fh:
        js = json.load(fh)
    return [(a, b, np.asarray(v, dtype=np.float64)) for (a, b), v in zip(js["ranges"], js["losses"])]


def _floor(name):
    path = os.path.join(GOLDEN, f"bf16_floor_{name}.json")
    if not os.path.exists(path):
        return None
    with open(path) as fh:
        return np.asarray(json.load(fh)["abs_err"], dtype=np.float64)


def _per_token_ok(d, floor, where):
    """max |d| <= 5e-2, or (when the storage floor exceeds 5e-2) d within 1.25x the floor's distribution."""
    if floor is None or floor.max() <= 5e-2:
        assert d.max() <= 5e-2, (where, d.max())
        return
    for q in (50, 90, 99):
        assert np.percentile(d, q) <= 1.25 * np.percentile(floor, q), (where, q, np.percentile(d, q),
                                                                       np.percentile(floor, q))
    assert d.max() <= 1.25 * floor.max(), (where, d.max(), floor.max())


@pytest.mark.parametrize("name", ["125m", "760m", "2.7b"])
def test_full_size_prefix_parity(name):
    from test_long_context_b200.context import upload_weights
    cfg = synth.get_config(name)
    w = synth.make_weights(cfg)
    toks = synth.tokens(cfg)
    gw = upload_weights(((n, w.arrays[n], w.bits.get(n)) for n in w.arrays), cfg.dtype)
    cache = {}
    full = _gpu_run(cfg, toks, gw, cache)
    T = cfg.T
    assert np.isnan(full[T - 1]) and np.all(np.isfinite(full[:T - 1]))
    if os.path.exists(os.path.join(GOLDEN, f"prefix_losses_{name}.json")):
        spans = _stored_prefix(name)
    else:  # no stored prefix: the oracle runs one chunk and a half here
        prefix = 1536
        ref = oracle.prefill(oracle.Model(cfg, w.arrays), toks[:prefix]).losses
        spans = [(0, prefix - 1, ref[:prefix - 1])]
    floor = _floor(name)
    B = cfg.b
    for a, b, ref in spans:
        d = np.abs(full[a:b] - ref)
        # per chunk: positions before the first update and after it are compared separately
        for c0 in range(a - a % B, b, B):
            lo, hi = max(a, c0), min(b, c0 + B)
            _per_token_ok(d[lo - a:hi - a], floor, (name, lo, hi))
        cm = np.abs(chunk_means(full[a:b], B) - chunk_means(ref, B))
        assert cm.max() <= 1e-2, (name, a, cm.max())
    if name == "2.7b":
        # properties at full size: determinism and causality
        again = _gpu_run(cfg, toks, gw, cache)
        np.testing.assert_array_equal(again, full)
        q = T - 1000
        t2 = toks.copy()
        t2[q:] = (t2[q:] + 1) % cfg.vocab
        other = _gpu_run(cfg, t2, gw, cache)
        np.testing.assert_array_equal(other[:q - 1], full[:q - 1])
        assert not np.array_equal(other[q - 1:T - 1], full[q - 1:T - 1])
    cache["ctx"].close()
