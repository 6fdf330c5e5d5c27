"""Several independent sequences prefilled at the same time, one context and
CUDA stream each (every document of a batch starts from W_init and adapts on
its own: reading notes by Zhongzhu Zhou, 算法 2): every sequence must get
exactly the losses and fast weights of a prefill that runs alone - the
contexts share the static weights and nothing else."""
import numpy as np
import pytest
import torch

import synth

pytestmark = pytest.mark.gpu

CFG = synth.ModelConfig("multi", n_layers=3, d_model=128, n_heads=2, head_dim=64, d_ff=256, vocab=1000,
                        n_updated=2, T=900, k=200, b=128, eta=0.5, dtype="bf16", seed=51)


def _run_alone(ctx, toks):
    ctx.reset()
    fast = ctx.fast_out_buffers()
    losses, fast = ctx.prefill(toks, fast_out=fast)
    return losses.clone(), [t.clone() for t in fast]


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_concurrent_contexts_match_solo_runs(dtype):
    from test_long_context_b200.context import Context, upload_weights
    cfg = CFG.with_(dtype=dtype)
    w = synth.make_weights(cfg)
    gw = upload_weights(((n, w.arrays[n], w.bits.get(n)) for n in w.arrays), cfg.dtype)
    n_seq = 3
    streams = [torch.cuda.Stream() for _ in range(n_seq)]
    ctxs = [Context(cfg, gw, stream=s) for s in streams]
    toks = [torch.from_numpy(synth.tokens(cfg, cfg.T - 37 * i, seed=cfg.seed + i)).cuda() for i in range(n_seq)]
    solo = [_run_alone(c, t) for c, t in zip(ctxs, toks)]
    torch.cuda.synchronize()
    # all at once, each on its own stream
    outs = []
    for c, t in zip(ctxs, toks):
        c.reset()
        fast = c.fast_out_buffers()
        losses, fast = c.prefill(t, fast_out=fast, sync=False)
        outs.append((losses, fast))
    for c in ctxs:
        c.sync()
    for (l1, f1), (l2, f2) in zip(solo, outs):
        assert torch.equal(l1, l2) or np.array_equal(l1.cpu().numpy(), l2.cpu().numpy(), equal_nan=True)
        for a, b in zip(f1, f2):
            assert torch.equal(a, b)
    for c in ctxs:
        c.close()
