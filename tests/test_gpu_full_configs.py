"""Parity at the full workload sizes, in the launch configuration bench.py
times (one sequence of T tokens through ttt_prefill).

The oracle cannot run a whole 128K-token prefill, so it runs a prefix: by
causality (算法 1 of the reading notes scores every position of a chunk
before that chunk's labels update W), the losses of positions 0 .. T'-2 of the full GPU
run equal those of a T'-token run, and W after the chunks that end before
T'-1 is the same.  T' covers one full chunk (so an SGD update happens) and
part of the next (scored with the updated weights).  At full size the GPU
run is also checked for properties that hold at any size: run-to-run
bit-identical losses, causality under a perturbed late token, finiteness.

Tolerances: bf16 mean chunk loss 1e-2 absolute and per-token loss 5e-2
absolute.  At 2.7B (32 blocks, d = 2560) the per-token bound is reached by
the bf16 rounding of the activations alone: rounding the same tensors to
bf16 in the fp64 CPU model (bf16_rounding_noise.py in this directory)
gives the same error distribution as the GPU at 125M, and at 2.7B a few
positions in a thousand land between 5e-2 and 6e-2 while the chunk means
stay within 1e-3.  There the per-token check is on the 99.5th percentile
(5e-2) plus a ceiling of 8e-2 on the maximum."""
import numpy as np
import pytest
import torch

import oracle
import synth

from ._gpu_helpers import chunk_means

pytestmark = pytest.mark.gpu


def _gpu_run(cfg, toks, weights_dev, ctx_cache):
    from test_long_context_b200.context import Context
    if "ctx" not in ctx_cache:
        ctx_cache["ctx"] = Context(cfg, weights_dev)
    ctx = ctx_cache["ctx"]
    ctx.reset()
    losses, _ = ctx.prefill(torch.from_numpy(np.asarray(toks, dtype=np.int32)).cuda())
    return losses.cpu().numpy().astype(np.float64)


@pytest.mark.parametrize("name,prefix", [("125m", 1536), ("760m", 1536), ("2.7b", 1536)])
def test_full_size_prefix_parity(name, prefix):
    from test_long_context_b200.context import upload_weights
    cfg = synth.get_config(name)
    w = synth.make_weights(cfg)
    toks = synth.tokens(cfg)
    gw = upload_weights(((n, w.arrays[n], w.bits.get(n)) for n in w.arrays), cfg.dtype)
    cache = {}
    full = _gpu_run(cfg, toks, gw, cache)
    T = cfg.T
    assert np.isnan(full[T - 1]) and np.all(np.isfinite(full[:T - 1]))
    ref = oracle.prefill(oracle.Model(cfg, w.arrays), toks[:prefix]).losses
    d = np.abs(full[:prefix - 1] - ref[:prefix - 1])
    if name == "2.7b":
        assert np.percentile(d, 99.5) <= 5e-2, np.percentile(d, 99.5)
        assert d.max() <= 8e-2, d.max()
    else:
        assert d.max() <= 5e-2, d.max()
    cm = np.abs(chunk_means(full[:prefix - 1], cfg.b) - chunk_means(ref[:prefix - 1], cfg.b))
    assert cm.max() <= 1e-2, cm.max()
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
