"""Parity across super-chunks of the fast-weight-free blocks.

The CUDA path runs the blocks without fast weights over super-chunks of
16 384 positions (their outputs depend on the tokens only), with their own
key/value rings of 16 384 + k slots (rounded up to 128) and a RoPE table per
super-chunk; the blocks with fast weights then run chunk by chunk.  A
sequence of 40 000 positions with b = 128 spans three super-chunks, so these
tests reach the second and third passes of the bottom rings (the ring wraps
at 16 768 slots here), the table rebase at 16 384 and 32 768, and windows
that straddle both boundaries.  Every per-token loss and the change of every
fast weight is compared with the oracle, which runs the plain chunk loop of
算法 1 (reading notes) with no super-chunks at all.

Tolerances are those of the other parity tests: fp32 per-token loss 1e-4
relative, W_final and W_final - W_init 1e-3 relative; bf16 per-token loss 5e-2
and chunk mean 1e-2 absolute, W_final - W_init 5e-2 relative."""
import numpy as np
import pytest

import synth

from ._gpu_helpers import chunk_means, rel, run_cuda, run_oracle

pytestmark = pytest.mark.gpu

# 3 blocks (2 without fast weights), d = 128 as 2 heads x 64, window 300
LONG = synth.ModelConfig("long", n_layers=3, d_model=128, n_heads=2, head_dim=64, d_ff=256, vocab=1000,
                         n_updated=1, T=40000, k=300, b=128, eta=0.1, dtype="f32", seed=23)
BOUNDARIES = (16384, 32768)


def _compare(cfg, fp32):
    w = synth.make_weights(cfg)
    toks = synth.tokens(cfg)
    L_gpu, W_gpu, _ = run_cuda(cfg, toks, w)
    r = run_oracle(cfg, toks, w)
    T = cfg.T
    assert np.isnan(L_gpu[T - 1])
    if fp32:
        err = np.abs(L_gpu[:T - 1] - r.losses[:T - 1]) / np.abs(r.losses[:T - 1])
        tol = 1e-4
    else:
        err = np.abs(L_gpu[:T - 1] - r.losses[:T - 1])
        tol = 5e-2
        cm = np.abs(chunk_means(L_gpu, cfg.b) - chunk_means(r.losses, cfg.b))
        assert cm.max() <= 1e-2, cm.max()
    # report the worst position of each super-chunk on failure
    spans = [(0, BOUNDARIES[0]), (BOUNDARIES[0], BOUNDARIES[1]), (BOUNDARIES[1], T - 1)]
    worst = {f"{a}-{b}": float(err[a:b].max()) for a, b in spans}
    assert err.max() <= tol, worst
    # the positions just past each boundary see keys from the previous super-chunk
    for p in BOUNDARIES:
        assert err[p:p + cfg.k].max() <= tol, (p, float(err[p:p + cfg.k].max()))
    for l in r.W:
        for n in r.W[l]:
            d_orc = r.W[l][n] - w.arrays[f"fast.{l}.{n}"]
            assert np.linalg.norm(d_orc) > 0
            if fp32:
                assert rel(W_gpu[l][n], r.W[l][n]) <= 1e-3, (l, n)
                assert rel(W_gpu[l][n] - w.arrays[f"fast.{l}.{n}"], d_orc) <= 1e-3, (l, n)
            else:
                assert rel(W_gpu[l][n] - w.arrays[f"fast.{l}.{n}"], d_orc) <= 5e-2, (l, n)


def test_three_super_chunks_fp32():
    _compare(LONG, fp32=True)


def test_three_super_chunks_bf16():
    """bf16 takes the tensor-core attention and GEMM kernels (head_dim 64,
    rings of whole 128-row tiles)."""
    _compare(LONG.with_(dtype="bf16"), fp32=False)
