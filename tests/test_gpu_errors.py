"""Error paths of the ttt_prefill contract (include/ttt.h), made on the host
side: no kernel is made to fault.

* ttt_prefill on a context that already ran a prefill (no ttt_reset between)
  returns TTT_ERR_STATE and enqueues nothing;
* a token id outside [0, vocab) is found on the device (the embedding reads
  row 0 instead and a flag is raised), ttt_sync returns TTT_ERR_INVALID_ARG
  and clears the flag, and after ttt_reset the same context reproduces a clean
  run bit for bit."""
import numpy as np
import pytest
import torch

import synth

pytestmark = pytest.mark.gpu

CFG = synth.ModelConfig("errs", n_layers=3, d_model=128, n_heads=2, head_dim=64, d_ff=256, vocab=1000,
                        n_updated=2, T=300, k=200, b=128, eta=0.5, dtype="bf16", seed=31)


def _ctx():
    from test_long_context_b200.context import Context, upload_weights
    w = synth.make_weights(CFG)
    gw = upload_weights(((n, w.arrays[n], w.bits.get(n)) for n in w.arrays), CFG.dtype)
    return Context(CFG, gw), gw


def test_prefill_twice_without_reset_is_a_state_error():
    from test_long_context_b200 import _lib as L
    ctx, _ = _ctx()
    toks = torch.from_numpy(synth.tokens(CFG)).cuda()
    first, _ = ctx.prefill(toks)
    first = first.cpu().numpy()
    with pytest.raises(L.TTTError) as e:
        ctx.prefill(toks)
    assert e.value.code == L.TTT_ERR_STATE
    ctx.sync()  # nothing was enqueued, nothing is pending
    ctx.reset()
    again, _ = ctx.prefill(toks)
    np.testing.assert_array_equal(again.cpu().numpy(), first)
    ctx.close()


@pytest.mark.parametrize("bad", [CFG.vocab, -1])
def test_bad_token_is_reported_and_the_context_recovers(bad):
    from test_long_context_b200 import _lib as L
    ctx, _ = _ctx()
    good = synth.tokens(CFG)
    clean, _ = ctx.prefill(torch.from_numpy(good).cuda())
    clean = clean.cpu().numpy()
    ctx.reset()
    t = good.copy()
    t[CFG.T // 2] = bad
    with pytest.raises(L.TTTError) as e:
        ctx.prefill(torch.from_numpy(t).cuda())  # asynchronous: the status arrives with ttt_sync
    assert e.value.code == L.TTT_ERR_INVALID_ARG
    assert "token" in str(e.value)
    ctx.sync()  # the flag was cleared by the failing sync
    ctx.reset()
    after, _ = ctx.prefill(torch.from_numpy(good).cuda())
    np.testing.assert_array_equal(after.cpu().numpy(), clean)
    ctx.close()
