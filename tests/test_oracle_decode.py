"""Pins of oracle.decode (greedy generation with periodic fast-weight
updates, 算法 3 of the reading notes), CPU only.

* eta = 0: no update ever changes W, so decoding is plain greedy decoding
  of the static model; it must give the tokens (and losses) of
  transformers' Qwen3 recomputing the whole sequence at every step — a
  library model, not the oracle;
* a generated chunk updates W exactly as the prefill does when the same
  tokens are read as a prompt (the pages' generation continues the same
  inner loop); with a prompt that ends inside a chunk, decoding until that
  chunk and the next are complete equals the prefill of the prompt plus the
  generated tokens, in fast weights and in every loss;
* all-zero LM head: every logit ties, so greedy takes id 0 every time, every
  loss is ln V, and W never moves (the gradient reaching W is zero);
* updates happen after the positions p with (p + 1) % b == 0, and only there."""
import math

import numpy as np
import pytest
import torch

import oracle
import synth

from . import _qwen3_pin as Q


def _cfg(micro_cfg, **kw):
    return micro_cfg.with_(**kw)


def test_eta_zero_decode_is_greedy_decoding_of_qwen3(micro_cfg):
    cfg = _cfg(micro_cfg, eta=0.0)
    w = synth.make_weights(cfg)
    prompt = synth.tokens(cfg)[:13]
    n_gen = 22
    r = oracle.decode(oracle.Model(cfg, w.arrays), prompt, n_gen)
    qm = Q.build(cfg.with_(T=64), w.arrays)
    seq = [int(t) for t in prompt]
    want_tok, want_loss = [], []
    for _ in range(n_gen):
        with torch.no_grad():
            z = qm(input_ids=torch.tensor([seq])).logits[0, -1]
        x = int(torch.argmax(z))
        want_tok.append(x)
        want_loss.append(float(torch.logsumexp(z, 0) - z[x]))
        seq.append(x)
    np.testing.assert_array_equal(r.tokens, want_tok)
    # transformers computes its RMSNorms in fp32 even in a double model: agreement to ~1e-7
    np.testing.assert_allclose(r.losses, want_loss, rtol=1e-6, atol=1e-6)


@pytest.mark.parametrize("T0", [13, 17])
def test_generated_chunks_update_like_the_prefill(micro_cfg, T0):
    cfg = _cfg(micro_cfg, eta=0.5)
    w = synth.make_weights(cfg)
    m = oracle.Model(cfg, w.arrays)
    prompt = synth.tokens(cfg)[:T0]
    b = cfg.b
    # decode until the chunk holding the prompt's end and the next one are complete
    end = (T0 // b + 2) * b                      # first position after them
    n_gen = end - T0
    r = oracle.decode(m, prompt, n_gen)
    assert r.updates == [p for p in range(T0, end) if (p + 1) % b == 0]
    seq = np.concatenate([prompt, r.tokens])
    # the prefill needs the target of position end-1 too: the next greedy token
    nxt = oracle.decode(m, prompt, n_gen + 1).tokens[-1]
    full = oracle.prefill(m, np.concatenate([seq, [nxt]]))
    for l in r.W:
        for n in r.W[l]:
            np.testing.assert_allclose(r.W[l][n], full.W[l][n], rtol=1e-11, atol=1e-13)
    # loss of position p-1 against generated token p, for every generated token
    np.testing.assert_allclose(r.losses, full.losses[T0 - 1:end - 1], rtol=1e-11, atol=1e-12)
    assert not all(np.array_equal(r.W[l][n], w.arrays[f"fast.{l}.{n}"]) for l in r.W for n in r.W[l])


def test_zero_head_decodes_lowest_id_and_ln_v(micro_cfg):
    cfg = _cfg(micro_cfg, eta=0.5)
    w = synth.make_weights(cfg)
    w.arrays["lm_head"] = np.zeros_like(w.arrays["lm_head"])
    r = oracle.decode(oracle.Model(cfg, w.arrays), synth.tokens(cfg)[:11], 20)
    assert (r.tokens == 0).all()
    np.testing.assert_allclose(r.losses, math.log(cfg.vocab), rtol=0, atol=1e-12)
    for l in r.W:
        for n in r.W[l]:
            np.testing.assert_array_equal(r.W[l][n], w.arrays[f"fast.{l}.{n}"])


def test_prompt_on_a_chunk_boundary(micro_cfg):
    """T % b == 0: the prefill already applied its last chunk (with b - 1
    targets); generation starts a new chunk at T."""
    cfg = _cfg(micro_cfg, eta=0.5)
    w = synth.make_weights(cfg)
    m = oracle.Model(cfg, w.arrays)
    b = cfg.b
    prompt = synth.tokens(cfg)[:2 * b]
    r = oracle.decode(m, prompt, b + 3)
    assert r.updates == [3 * b - 1]
    pre = oracle.prefill(m, prompt)
    # the first generated token comes from the logits of position T-1 scored before its chunk's update
    assert r.tokens[0] == int(np.argmax(pre.z_last))
