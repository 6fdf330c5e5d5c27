"""Greedy generation with periodic fast-weight updates (ttt_decode /
ttt_decode_step, 算法 3 of the reading notes) against oracle.decode on the
same seeded prompts.

fp32: every generated token must be the oracle's (the argmax is an integer
decision taken on fp32 logits whose error is ~1e-6, far below the gaps
between the largest logits here), and every loss within 1e-4 relative;
the prompts end inside a chunk and on a chunk boundary, and generation runs
across two updates.  bf16: tokens must agree up to the first position where
the oracle's top two logits lie within the bf16 noise of the logits (2e-2);
there the GPU's pick must be one of those near-ties; losses up to that point
within 5e-2.  Also: decoding continues the prefill's inner loop, so a
prefill of the prompt plus the generated tokens gives the decode's losses
(GPU against GPU), and ttt_decode_step gives the same tokens as ttt_decode."""
import numpy as np
import pytest
import torch

import oracle
import synth

pytestmark = pytest.mark.gpu

SMALL = synth.ModelConfig("dec", n_layers=3, d_model=128, n_heads=2, head_dim=64, d_ff=256, vocab=1000,
                          n_updated=2, T=700, k=200, b=128, eta=0.5, dtype="f32", seed=41)


def _setup(cfg):
    from test_long_context_b200.context import Context, upload_weights
    w = synth.make_weights(cfg)
    gw = upload_weights(((n, w.arrays[n], w.bits.get(n)) for n in w.arrays), cfg.dtype)
    return w, gw, Context(cfg, gw)


def _gpu_decode(ctx, prompt, n_gen):
    ctx.reset()
    ctx.prefill(torch.from_numpy(np.asarray(prompt, dtype=np.int32)).cuda())
    toks, losses = ctx.decode(n_gen, losses=torch.empty(n_gen, device="cuda"))
    return toks.cpu().numpy().astype(np.int64), losses.cpu().numpy().astype(np.float64)


@pytest.mark.parametrize("T0,over", [(300, {}), (256, {}), (200, dict(k=64)), (300, dict(head_dim=32, n_heads=4))])
def test_decode_fp32_matches_oracle(T0, over):
    cfg = SMALL.with_(**over)
    w, _, ctx = _setup(cfg)
    prompt = synth.tokens(cfg)[:T0]
    n_gen = (T0 // cfg.b + 3) * cfg.b - T0 + 5     # two updates and a few tokens past the second
    ref = oracle.decode(oracle.Model(cfg, w.arrays), prompt, n_gen)
    assert len(ref.updates) >= 2
    assert ref.gaps.min() > 1e-4, "near-tie in the fp32 case: pick another seed"
    toks, losses = _gpu_decode(ctx, prompt, n_gen)
    np.testing.assert_array_equal(toks, ref.tokens)
    np.testing.assert_allclose(losses, ref.losses, rtol=1e-4, atol=0)
    # decoding continues the prefill's loop: with a prompt that ends inside a
    # chunk, the prefill of prompt + generated tokens scores them alike
    # (at T0 % b == 0 the prompt's last chunk was applied with b - 1 targets)
    if T0 % cfg.b:
        seq = np.concatenate([prompt, toks]).astype(np.int32)
        ctx.reset()
        full, _ = ctx.prefill(torch.from_numpy(seq).cuda())
        full = full.cpu().numpy().astype(np.float64)
        np.testing.assert_allclose(full[T0 - 1:T0 - 1 + n_gen], losses, rtol=1e-4, atol=0)
    ctx.close()


def test_decode_step_equals_decode():
    cfg = SMALL
    _, _, ctx = _setup(cfg)
    prompt = synth.tokens(cfg)[:200]
    n = 70
    toks, _ = _gpu_decode(ctx, prompt, n)
    ctx.reset()
    ctx.prefill(torch.from_numpy(prompt.astype(np.int32)).cuda())
    out = torch.empty(n, device="cuda", dtype=torch.int32)
    for i in range(n):
        ctx.decode_step(out[i:i + 1], sync=False)
    ctx.sync()
    np.testing.assert_array_equal(out.cpu().numpy(), toks)
    ctx.close()


def test_decode_needs_a_prefill():
    from test_long_context_b200 import _lib as L
    _, _, ctx = _setup(SMALL)
    with pytest.raises(L.TTTError) as e:
        ctx.decode(3)
    assert e.value.code == L.TTT_ERR_STATE
    ctx.close()


@pytest.mark.parametrize("T0", [300, 256])
def test_decode_bf16_matches_oracle_until_a_near_tie(T0):
    cfg = SMALL.with_(dtype="bf16")
    w, _, ctx = _setup(cfg)
    prompt = synth.tokens(cfg)[:T0]
    n_gen = (T0 // cfg.b + 3) * cfg.b - T0 + 5
    ref = oracle.decode(oracle.Model(cfg, w.arrays), prompt, n_gen)
    toks, losses = _gpu_decode(ctx, prompt, n_gen)
    diff = np.nonzero(toks != ref.tokens)[0]
    upto = diff[0] if len(diff) else n_gen
    if len(diff):
        i = diff[0]
        assert ref.gaps[i] <= 2e-2, (i, ref.gaps[i])
    assert np.abs(losses[:upto] - ref.losses[:upto]).max() <= 5e-2
    # the comparison must reach past at least one update unless a near-tie comes first
    if upto < ref.updates[0] - T0 + 2:
        assert ref.gaps[:upto + 1].min() <= 2e-2
    ctx.close()
