"""ttt_prefill (CUDA, through the C ABI) vs the oracle on the same seeded
inputs.  Tolerances: fp32 per-token loss 1e-4 relative, final fast weights
1e-3 relative (also on W_final - W_init); bf16 mean chunk loss 1e-2
absolute, per-token loss 5e-2 absolute, fast-weight change 5e-2 relative
(bf16 operands carry ~4e-3 relative rounding into each gradient product)."""
import numpy as np
import pytest

import synth

from ._gpu_helpers import chunk_means, rel, run_cuda, run_oracle

pytestmark = pytest.mark.gpu


def _check_fp32(cfg, toks, w=None):
    L_gpu, W_gpu, _ = run_cuda(cfg, toks, w)
    r = run_oracle(cfg, toks, w)
    T = len(toks)
    assert np.isnan(L_gpu[T - 1]) and np.isnan(r.losses[T - 1])
    err = np.abs(L_gpu[:T - 1] - r.losses[:T - 1]) / np.abs(r.losses[:T - 1])
    assert err.max() <= 1e-4, err.max()
    w0 = (w or synth.make_weights(cfg)).arrays
    for l in r.W:
        for n in r.W[l]:
            assert rel(W_gpu[l][n], r.W[l][n]) <= 1e-3
            d_orc = r.W[l][n] - w0[f"fast.{l}.{n}"]
            if np.linalg.norm(d_orc) > 0:
                assert rel(W_gpu[l][n] - w0[f"fast.{l}.{n}"], d_orc) <= 1e-3, (l, n)


def _check_bf16(cfg, toks, w=None, dw_tol=5e-2):
    w = w or synth.make_weights(cfg)
    L_gpu, W_gpu, _ = run_cuda(cfg, toks, w)
    r = run_oracle(cfg, toks, w)
    T = len(toks)
    assert np.isnan(L_gpu[T - 1])
    d = np.abs(L_gpu[:T - 1] - r.losses[:T - 1])
    assert d.max() <= 5e-2, d.max()
    cm = np.abs(chunk_means(L_gpu, cfg.b) - chunk_means(r.losses, cfg.b))
    assert cm.max() <= 1e-2, cm.max()
    for l in r.W:
        for n in r.W[l]:
            d_orc = r.W[l][n] - w.arrays[f"fast.{l}.{n}"]
            if np.linalg.norm(d_orc) > 0:
                assert rel(W_gpu[l][n] - w.arrays[f"fast.{l}.{n}"], d_orc) <= dw_tol, (l, n)


def test_tiny_fp32_full_config():
    """The tiny fp32 workload at full size (T=4096, k=1024, b=256)."""
    cfg = synth.get_config("tiny")
    _check_fp32(cfg, synth.tokens(cfg))


SMALL = synth.ModelConfig("small", n_layers=3, d_model=128, n_heads=2, head_dim=64, d_ff=256, vocab=1000,
                          n_updated=2, T=700, k=200, b=128, eta=0.5, dtype="f32", seed=11)


@pytest.mark.parametrize("over", [dict(), dict(T=640), dict(k=64), dict(k=5000), dict(b=1, T=40),
                                  dict(n_updated=3), dict(head_dim=32, n_heads=4), dict(head_dim=80, n_heads=2,
                                  d_model=160, d_ff=192)])
def test_small_fp32_variants(over):
    """Ragged last chunk, T % b == 0, k < b, k >= T, b = 1, every block
    updated, other head sizes."""
    cfg = SMALL.with_(**over)
    _check_fp32(cfg, synth.tokens(cfg))


@pytest.mark.parametrize("over", [dict(), dict(T=640), dict(k=64), dict(n_updated=1), dict(head_dim=80, n_heads=2,
                                  d_model=160, d_ff=192), dict(head_dim=96, n_heads=2, d_model=192, d_ff=256)])
def test_small_bf16_variants(over):
    cfg = SMALL.with_(dtype="bf16", **over)
    _check_bf16(cfg, synth.tokens(cfg))


def _norm_gains_away_from_one(w, seed=5):
    """The synthetic weights start every RMSNorm gain at 1, where a gain
    applied to the wrong tensor (q vs k, attention vs MLP norm) or left out
    of a backward changes nothing; draw them as 1 + 0.3 N(0, 1) instead.
    Gains are fp32 on both sides in either dtype."""
    rng = np.random.default_rng(seed)
    for name in w.arrays:
        if name.endswith("norm"):
            w.arrays[name] = (1.0 + 0.3 * rng.standard_normal(w.arrays[name].shape)).astype(np.float32)
    return w


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_small_with_norm_gains_away_from_one(dtype):
    cfg = SMALL.with_(dtype=dtype)
    w = _norm_gains_away_from_one(synth.make_weights(cfg))
    if dtype == "f32":
        _check_fp32(cfg, synth.tokens(cfg), w)
    else:
        _check_bf16(cfg, synth.tokens(cfg), w)
