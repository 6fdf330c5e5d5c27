"""Shared helpers of the GPU parity tests: run the CUDA path and the oracle
on the same seeded inputs."""
import numpy as np
import torch

import oracle
import synth


def run_cuda(cfg, toks, weights=None, **ctx_kw):
    from test_long_context_b200.context import Context, upload_weights
    w = weights if weights is not None else synth.make_weights(cfg)
    gw = upload_weights(((n, w.arrays[n], w.bits.get(n)) for n in w.arrays), cfg.dtype)
    ctx = Context(cfg, gw, **ctx_kw)
    fast = ctx.fast_out_buffers()
    losses, fast = ctx.prefill(torch.from_numpy(np.asarray(toks, dtype=np.int32)).cuda(), fast_out=fast)
    out = losses.cpu().numpy().astype(np.float64), {l: {k: v.cpu().numpy().astype(np.float64) for k, v in d.items()}
                                                     for l, d in ctx.fast_dict(fast).items()}
    launches = ctx.launch_count()
    ctx.close()
    return out[0], out[1], launches


def run_oracle(cfg, toks, weights=None, **kw):
    w = weights if weights is not None else synth.make_weights(cfg)
    return oracle.prefill(oracle.Model(cfg, w.arrays), toks, **kw)


def rel(a, b):
    return float(np.linalg.norm(a - b) / max(np.linalg.norm(b), 1e-300))


def chunk_means(losses, b):
    T = len(losses)
    return np.array([np.nanmean(losses[c:c + b]) for c in range(0, T, b)])
