"""The outer-loop meta-gradient on the GPU (ttt_op_meta_grad) against the
fp64 oracle (oracle/meta_grad.py) on the same seeded fp32 inputs: eq. (7) of
the reading notes (End-to-End Test-Time Training for Long Context, §4) for a
fast MLP in the last block.  Shapes span several tiles of the fp32 GEMM
(64 x 128) with ragged tails; the cases include rows and a whole chunk
without a target, one chunk, eta = 0, and a step size large enough that the
Hessian term carries most of the result."""
import numpy as np
import pytest
import torch

from oracle import meta_grad as M

pytestmark = pytest.mark.gpu

EPS = 1e-5
# fp32 against fp64: a CPU fp32 run of the oracle's own steps differs by
# about 1e-6 of the largest entry; the GPU's accumulation order adds a little
GRAD_TOL = 2e-4
LOSS_TOL = 1e-4


def _inputs(seed, N, b, d, f, V, drop=()):
    rng = np.random.default_rng(seed)
    h = rng.standard_normal((N * b, d)).astype(np.float32)
    r = rng.standard_normal((N * b, d)).astype(np.float32)
    tgt = rng.integers(0, V, N * b).astype(np.int32)
    for i in drop:
        tgt[i] = -1
    tgt[-1] = -1  # the sequence's last position has no next token
    W = ((rng.standard_normal((f, d)) / np.sqrt(d)).astype(np.float32),
         (rng.standard_normal((f, d)) / np.sqrt(d)).astype(np.float32),
         (rng.standard_normal((d, f)) / np.sqrt(f)).astype(np.float32))
    gf = (1 + 0.2 * rng.standard_normal(d)).astype(np.float32)
    head = (1.5 * rng.standard_normal((V, d)) / np.sqrt(d)).astype(np.float32)
    return h, r, tgt, W, gf, head


def _first_order(h, r, tgt, W, gf, head, eta, b):
    """The same recursion with the Hessian term left out (to show that the
    cases below depend on it)."""
    N = len(tgt) // b
    rows = [slice(c * b, (c + 1) * b) for c in range(N)]

    def lg(c, Wc):
        fw = M.chunk_forward(h[rows[c]].astype(np.float64), r[rows[c]].astype(np.float64), tgt[rows[c]], Wc,
                             gf.astype(np.float64), head.astype(np.float64), EPS)
        return fw["A"], M.chunk_grad(fw, Wc, gf.astype(np.float64), head.astype(np.float64))[0]

    g, _, _ = M.meta_grad(N, W, eta, lg, lambda c, Wc, v: tuple(np.zeros_like(x) for x in v))
    return g


def _gpu(h, r, tgt, W, gf, head, eta, b):
    from test_long_context_b200 import ops
    dev = lambda a: torch.from_numpy(np.ascontiguousarray(a)).cuda()
    out = [torch.full(w.shape, float("nan"), device="cuda") for w in W]
    losses = torch.full((len(tgt),), 7.0, device="cuda")
    ops.meta_grad(dev(h), dev(r), dev(tgt), *[dev(w) for w in W], dev(gf), dev(head), EPS, eta, b, *out,
                  losses=losses)
    ops.sync()
    return [o.cpu().numpy().astype(np.float64) for o in out], losses.cpu().numpy().astype(np.float64)


CASES = [
    # seed, chunks, b, d, f, V, eta, rows without a target
    (1, 4, 100, 136, 200, 1000, 1.0, (5, 17)),
    (2, 4, 100, 136, 200, 1000, 4.0, ()),
    (3, 3, 37, 72, 100, 333, 1.0, tuple(range(37, 74))),   # chunk 1 has no target at all
    (4, 1, 130, 64, 256, 517, 0.7, (0,)),
    (5, 5, 64, 128, 128, 700, 0.0, ()),
]


@pytest.mark.parametrize("case", CASES, ids=lambda c: f"N{c[1]}-b{c[2]}-d{c[3]}-f{c[4]}-V{c[5]}-eta{c[6]}")
def test_meta_grad_matches_oracle(case):
    seed, N, b, d, f, V, eta, drop = case
    h, r, tgt, W, gf, head = _inputs(seed, N, b, d, f, V, drop)
    want, L, rows = M.meta_grad_top_mlp(h, r, tgt, W, gf, head, eta, EPS, b)
    got, losses = _gpu(h, r, tgt, W, gf, head, eta, b)
    for g, w in zip(got, want):
        assert np.isfinite(g).all()
        assert np.abs(g - w).max() <= GRAD_TOL * np.abs(w).max()
    assert np.array_equal(np.isnan(losses), np.isnan(rows))
    ok = ~np.isnan(rows)
    assert np.abs(losses[ok] - rows[ok]).max() <= LOSS_TOL * max(1.0, np.abs(rows[ok]).max())
    if eta > 0 and N > 1:
        fo = _first_order(h, r, tgt, W, gf, head, eta, b)
        assert max(np.abs(a - c).max() / np.abs(a).max() for a, c in zip(want, fo)) > 50 * GRAD_TOL


def test_meta_grad_is_deterministic():
    h, r, tgt, W, gf, head = _inputs(6, 3, 96, 136, 200, 900)
    a, la = _gpu(h, r, tgt, W, gf, head, 1.5, 96)
    b, lb = _gpu(h, r, tgt, W, gf, head, 1.5, 96)
    for x, y in zip(a, b):
        assert np.array_equal(x, y)
    assert np.array_equal(la, lb, equal_nan=True)


def test_target_out_of_range_is_reported_and_counts_as_none():
    from test_long_context_b200 import _lib as L
    from test_long_context_b200 import ops
    N, b, d, f, V = 2, 40, 64, 128, 300
    h, r, tgt, W, gf, head = _inputs(7, N, b, d, f, V)
    bad = tgt.copy()
    bad[3] = V  # outside [0, V)
    dev = lambda a: torch.from_numpy(np.ascontiguousarray(a)).cuda()
    out = [torch.empty(w.shape, device="cuda") for w in W]
    losses = torch.empty(N * b, device="cuda")
    ops.meta_grad(dev(h), dev(r), dev(bad), *[dev(w) for w in W], dev(gf), dev(head), EPS, 0.5, b, *out,
                  losses=losses)
    with pytest.raises(L.TTTError) as e:
        ops.sync()
    assert e.value.code == L.TTT_ERR_INVALID_ARG
    assert np.isnan(losses[3].item())
    none = tgt.copy()
    none[3] = -1
    want, _, _ = M.meta_grad_top_mlp(h, r, none, W, gf, head, 0.5, EPS, b)
    got = [o.cpu().numpy().astype(np.float64) for o in out]
    for g, w in zip(got, want):
        assert np.abs(g - w).max() <= GRAD_TOL * np.abs(w).max()
    ops.sync()  # the record was cleared


def test_meta_grad_rejects_a_small_work_array():
    from test_long_context_b200 import _lib as L
    from test_long_context_b200 import ops
    h, r, tgt, W, gf, head = _inputs(8, 2, 16, 32, 64, 50)
    dev = lambda a: torch.from_numpy(np.ascontiguousarray(a)).cuda()
    out = [torch.empty(w.shape, device="cuda") for w in W]
    work = torch.empty(ops.meta_grad_work(2, 16, 32, 64, 50) - 1, device="cuda")
    with pytest.raises(L.TTTError) as e:
        ops.meta_grad(dev(h), dev(r), dev(tgt), *[dev(w) for w in W], dev(gf), dev(head), EPS, 0.5, 16, *out,
                      work=work)
    assert e.value.code == L.TTT_ERR_INVALID_ARG
