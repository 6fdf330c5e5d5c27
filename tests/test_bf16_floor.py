"""Pins of oracle/bf16_floor.py, the fp64 forward with the bf16 pipeline's
storage roundings (CPU only).

* bf16_round agrees bit for bit with torch's float32 -> bfloat16 conversion
  (round to nearest, ties to even), ties and subnormal-range values included;
* with no rounding site the floor forward is the oracle's forward
  (oracle.static_losses) to fp64 rounding;
* each rounding site changes the losses (none is silently skipped), and the
  total stays at the size bf16 storage implies on a small model;
* the stored 2.7B floor (tests/golden/bf16_floor_2.7b.json) exceeds 5e-2 at
  some position: the per-token bound read as a maximum is below what bf16
  storage at these points allows at that depth."""
import json
import os

import numpy as np
import pytest
import torch

import oracle
import synth
from oracle import bf16_floor as F

HERE = os.path.dirname(os.path.abspath(__file__))
CFG = synth.ModelConfig("floor", n_layers=2, d_model=64, n_heads=2, head_dim=32, d_ff=128, vocab=256,
                        n_updated=1, T=96, k=40, b=96, eta=0.0, dtype="bf16", seed=0xF100)


def test_bf16_round_matches_torch():
    rng = np.random.default_rng(1)
    x = np.concatenate([rng.standard_normal(4096) * 10.0 ** rng.integers(-30, 30, 4096),
                        rng.standard_normal(512) * 1e-39])
    # exact ties: a bf16 value plus half an ulp (low 16 bits = 0x8000)
    base = rng.standard_normal(512).astype(np.float32).view(np.uint32) & np.uint32(0xFFFF0000)
    ties = (base | np.uint32(0x8000)).view(np.float32)
    x = np.concatenate([x, ties.astype(np.float64)])
    ref = torch.from_numpy(x.astype(np.float32)).to(torch.bfloat16).to(torch.float64).numpy()
    np.testing.assert_array_equal(F.bf16_round(x), ref)


@pytest.fixture(scope="module")
def model_toks():
    w = synth.make_weights(CFG)
    return oracle.Model(CFG, w.arrays), synth.tokens(CFG)


def test_no_site_is_the_oracle_forward(model_toks):
    m, toks = model_toks
    n = CFG.T - 1
    got = F.forward_losses(m, oracle.init_fast(m), toks, n, ())
    ref = oracle.static_losses(m, toks)[:n]
    np.testing.assert_allclose(got, ref, rtol=0, atol=1e-12)


@pytest.mark.parametrize("site", F.SITES)
def test_every_site_rounds_something(model_toks, site):
    m, toks = model_toks
    d = F.floor(m, toks, CFG.T - 1, sites=(site,))
    assert d.max() > 0, site
    assert d.max() < 2e-2, (site, d.max())


def test_all_sites_small_model(model_toks):
    m, toks = model_toks
    d = F.floor(m, toks, CFG.T - 1)
    assert 1e-5 < d.mean() < 1e-2, d.mean()


def test_stored_2_7b_floor_exceeds_the_per_token_bound():
    path = os.path.join(HERE, "golden", "bf16_floor_2.7b.json")
    if not os.path.exists(path):
        pytest.skip("golden floor not generated")
    with open(path) as fh:
        js = json.load(fh)
    d = np.asarray(js["abs_err"])
    assert len(d) == js["positions"]
    assert d.max() > 5e-2
    assert np.percentile(d, 50) < 5e-2
