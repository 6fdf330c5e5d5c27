"""Planted mistakes in the CPU oracle must each fail at least one pin.

Each mutation replaces one oracle step by a plausible wrong version (a sign,
an index, a dropped term, a missing scale) for the duration of one test; the
pins of test_oracle_pins.py are then run on the micro model until one fails.
A mutation that no pin catches fails this test: it would mean that part of
the oracle is not pinned to anything outside itself."""
import math

import numpy as np
import pytest

import synth
from oracle import ttt_oracle as O

from . import test_oracle_pins as P

CFG = synth.ModelConfig("micro", n_layers=2, d_model=32, n_heads=2, head_dim=16, d_ff=64, vocab=64, n_updated=1,
                        T=40, k=12, b=8, eta=0.05, dtype="f32", seed=0x5EED)


def _rope_wrong_sign(orig):
    def f(x, cos, sin):
        return orig(x, cos, -sin)
    return f


def _rope_bwd_wrong_sign(orig):
    def f(dy, cos, sin):
        return orig(dy, cos, -sin)
    return f


def _window_one_too_wide(orig):
    def f(qpos, kpos, k):
        return orig(qpos, kpos, k + 1)
    return f


def _rmsnorm_bwd_drops_term(orig):
    def f(x, r, g, dy):
        return r * dy * g
    return f


def _silu_derivative_wrong(orig):
    def f(dy, h, g, u, a, wg, wu, wd, need_dh=True):
        sg = O.sigmoid(g)
        da = dy @ wd
        dg = da * u * sg                       # missing the (1 + g (1 - s)) factor
        du = da * g * sg
        dh = dg @ wg + du @ wu if need_dh else None
        return dh, (dg.T @ h, du.T @ h, dy.T @ a)
    return f


def _softmax_bwd_drops_row_term(orig):
    def f(do, q, K, V, P_, hd):
        scale = 1.0 / math.sqrt(hd)
        dP = np.einsum("nhe,mhe->hnm", do, V)
        dV = np.einsum("hnm,nhe->mhe", P_, do)
        dS = P_ * dP                           # missing - sum(dP * P)
        return (np.einsum("hnm,mhe->nhe", dS, K) * scale, np.einsum("hnm,nhe->mhe", dS, q) * scale, dV)
    return f


def _attention_unscaled(orig):
    def f(q, K, V, qpos, kpos, k):
        return orig(q * math.sqrt(q.shape[-1]), K, V, qpos, kpos, k)
    return f


def _gradient_sign_flipped(orig):
    def f(model, W, fwd, weights):
        G = orig(model, W, fwd, weights)
        return {l: {n: -g for n, g in d.items()} for l, d in G.items()}
    return f


def _norm_gain_ignored(orig):
    def f(x, g, eps):
        return orig(x, np.ones_like(g), eps)
    return f


def _norm_bwd_gain_ignored(orig):
    def f(x, r, g, dy):
        return orig(x, r, np.ones_like(g), dy)
    return f


def _rope_theta_doubled(orig):
    def f(pos, hd, theta):
        return orig(pos, hd, 2.0 * theta)
    return f


def _next_key_visible(orig):
    def f(qpos, kpos, k):
        qp = np.asarray(qpos)[:, None]
        kp = np.asarray(kpos)[None, :]
        return (kp <= qp + 1) & (kp > qp - k)
    return f


def _rope_adjacent_pairs(orig):
    def f(x, cos, sin):
        c, s = cos[:, None, :], sin[:, None, :]
        x1, x2 = x[..., 0::2], x[..., 1::2]
        y = np.empty_like(x)
        y[..., 0::2] = x1 * c - x2 * s
        y[..., 1::2] = x2 * c + x1 * s
        return y
    return f


def _norm_eps_wrong(orig):
    def f(x, g, eps):
        return orig(x, g, 100.0 * eps)
    return f


def _ce_target_shifted(orig):
    def f(z, targets):
        return orig(z, (np.asarray(targets) + 1) % z.shape[-1])
    return f


MUTATIONS = {
    "rope rotates the wrong way": ("rope", _rope_wrong_sign),
    "rope backward rotates the wrong way": ("rope_bwd", _rope_bwd_wrong_sign),
    "window admits one key too many": ("window_mask", _window_one_too_wide),
    "rmsnorm backward drops the mean term": ("rmsnorm_bwd", _rmsnorm_bwd_drops_term),
    "SiLU derivative missing a factor": ("swiglu_bwd", _silu_derivative_wrong),
    "softmax backward drops the row term": ("swa_bwd", _softmax_bwd_drops_row_term),
    "attention scale missing": ("swa", _attention_unscaled),
    "SGD step climbs the loss": ("backward_chunk", _gradient_sign_flipped),
    "cross-entropy scores the wrong target": ("log_softmax_ce", _ce_target_shifted),
    "RMSNorm forward ignores its gain": ("rmsnorm", _norm_gain_ignored),
    "RMSNorm backward ignores its gain": ("rmsnorm_bwd", _norm_bwd_gain_ignored),
    "RoPE base theta doubled": ("rope_tables", _rope_theta_doubled),
    "causal mask lets the next key in": ("window_mask", _next_key_visible),
    "RoPE pairs adjacent elements": ("rope", _rope_adjacent_pairs),
    "RMSNorm eps 100x too large": ("rmsnorm", _norm_eps_wrong),
}

PINS = {
    "forward vs Qwen3 (k = 12)": lambda: P.test_forward_matches_qwen3_sliding_window(CFG, 12),
    "backward vs central differences (chunk 2)": lambda: P.test_backward_matches_central_differences(CFG, 2, False),
    "eq. (3) toy, b = 1": lambda: P.test_toy_bigram_per_token_update_eq3(CFG),
    "eq. (9) chunk gradient": lambda: P.test_chunk_gradient_is_mean_of_token_gradients_eq9(CFG),
    "zero head: ln V": lambda: P.test_zero_head_gives_ln_V_and_zero_gradient(CFG),
    "forward vs Qwen3, random norm gains": lambda: P.test_forward_matches_qwen3_with_random_norm_gains(CFG),
    "central differences, random norm gains": lambda: P.test_backward_matches_central_differences(CFG, 2, True),
}


@pytest.mark.parametrize("name", sorted(MUTATIONS))
def test_a_pin_catches_the_planted_mistake(name, monkeypatch):
    attr, make = MUTATIONS[name]
    monkeypatch.setattr(O, attr, make(getattr(O, attr)))
    caught = None
    for pin, run in PINS.items():
        try:
            run()
        except AssertionError:
            caught = pin
            break
    assert caught is not None, f"no pin fails when: {name}"


def test_every_pin_passes_on_the_unmutated_oracle():
    """Control: the pins used above pass as they stand, so a failure under a
    mutation comes from the planted mistake."""
    for run in PINS.values():
        run()
