"""Sliding-window attention kernels (op-level C ABI) vs the oracle's
attention and its backward, on ring buffers that wrap."""
import math

import numpy as np
import pytest
import torch

from oracle import ttt_oracle as O

pytestmark = pytest.mark.gpu


def _case(H, hd, n, p0, window, ring, dtype, seed):
    g = torch.Generator().manual_seed(seed)
    P = p0 + n
    Kall = torch.randn(P, H * hd, generator=g, dtype=torch.float64)
    Vall = torch.randn(P, H * hd, generator=g, dtype=torch.float64)
    q = torch.randn(n, H * hd, generator=g, dtype=torch.float64)
    dout = torch.randn(n, H * hd, generator=g, dtype=torch.float64)
    tdt = torch.bfloat16 if dtype == "bf16" else torch.float32
    # round to the storage type so both sides see the same values
    Kall, Vall, q, dout = (t.to(tdt).double() for t in (Kall, Vall, q, dout))
    kr = torch.zeros(ring, H * hd, dtype=torch.float64)
    vr = torch.zeros(ring, H * hd, dtype=torch.float64)
    for j in range(P):
        kr[j % ring] = Kall[j]
        vr[j % ring] = Vall[j]
    return Kall, Vall, q, dout, kr, vr, tdt


CASES = [(100, 350, 120, 256), (64, 0, 1000, 64), (37, 5, 1, 64), (130, 900, 64, 200), (300, 1000, 700, 1152),
         (129, 0, 5000, 256), (200, 4000, 4096, 4352), (1, 77, 3, 128), (256, 2048, 128, 384),
         (384, 1024, 300, 1792), (200, 512, 64, 896)]


@pytest.mark.parametrize("impl", ["f32", "bf16-simt", "bf16"])
@pytest.mark.parametrize("hd", [32, 64, 80, 96, 128])
@pytest.mark.parametrize("n,p0,window,ring", CASES)
def test_swa_forward_backward_vs_oracle(impl, hd, n, p0, window, ring):
    """bf16 with ring % 128 == 0 and head_dim in {64, 80, 96, 128} runs the
    tcgen05 kernel; the other cases the SIMT kernel."""
    dtype = "f32" if impl == "f32" else "bf16"
    from test_long_context_b200 import ops
    H = 2
    Kall, Vall, q, dout, kr, vr, tdt = _case(H, hd, n, p0, window, ring, dtype, seed=hd + n)
    qpos = np.arange(p0, p0 + n)
    ks = max(0, p0 - window + 1)
    kpos = np.arange(ks, p0 + n)
    Kw = Kall[ks:p0 + n].numpy().reshape(-1, H, hd)
    Vw = Vall[ks:p0 + n].numpy().reshape(-1, H, hd)
    qq = q.numpy().reshape(n, H, hd)
    o_ref, P = O.swa(qq, Kw, Vw, qpos, kpos, window)
    s = np.einsum("nhe,mhe->hnm", qq, Kw) / math.sqrt(hd)
    s = np.where(O.window_mask(qpos, kpos, window)[None], s, -np.inf)
    lse_ref = np.log(np.exp(s - s.max(-1, keepdims=True)).sum(-1)) + s.max(-1)
    dq_ref, dK, dV = O.swa_bwd(dout.numpy().reshape(n, H, hd), qq, Kw, Vw, P, hd)
    off = p0 - ks
    dk_ref, dv_ref = dK[off:off + n], dV[off:off + n]

    cu = lambda t: t.to(tdt).cuda().contiguous()
    qd, krd, vrd, dd = cu(q), cu(kr), cu(vr), cu(dout)
    o = torch.empty(n, H * hd, device="cuda", dtype=tdt)
    lse = torch.empty(H, n, device="cuda")
    ops.swa_forward(qd, krd, vrd, H, hd, p0, window, o, lse, force_simt=(impl == "bf16-simt"))
    dq = torch.empty_like(o)
    dk = torch.empty_like(o)
    dv = torch.empty_like(o)
    D = torch.empty(H * n, device="cuda")
    ops.swa_backward(qd, krd, vrd, H, hd, p0, window, o, lse, dd, dq, dk, dv, D, force_simt=(impl == "bf16-simt"))
    ops.sync()
    tol = 2e-2 if dtype == "bf16" else 1e-5

    def close(a, b, name):
        a = a.double().cpu().numpy().reshape(b.shape)
        err = np.abs(a - b).max()
        assert err <= tol * max(1.0, np.abs(b).max()), (name, err)

    close(o, o_ref, "o")
    close(lse, lse_ref, "lse")
    close(dq, dq_ref, "dq")
    close(dk, dk_ref, "dk")
    close(dv, dv_ref, "dv")


@pytest.mark.parametrize("hd", [64, 80, 96, 128])
def test_tc_forward_rescale_on_some_rows(hd):
    """Keys planted as 2x the query of a few rows make those rows' running
    max jump by far more than 2^8 in a late key tile while the other rows of
    the same warp keep theirs: the warp-collective O rescale in TMEM must
    serve both kinds of rows."""
    from test_long_context_b200 import ops
    H, n, p0, window, ring = 2, 256, 1024, 1024, 2048
    Kall, Vall, q, dout, kr, vr, tdt = _case(H, hd, n, p0, window, ring, "bf16", seed=5)
    rows = [130, 131, 140, 200, 255]   # some rows of warps 0 and 1 of the second query tile
    for t, r in enumerate(rows):
        j = p0 + 128 + t                  # visible to every planted row (j <= p0 + r)
        Kall[j] = 2.0 * q[r]
        kr[j % ring] = Kall[j]
    Kall, kr = Kall.to(tdt).double(), kr.to(tdt).double()
    qpos = np.arange(p0, p0 + n)
    ks = max(0, p0 - window + 1)
    kpos = np.arange(ks, p0 + n)
    Kw = Kall[ks:p0 + n].numpy().reshape(-1, H, hd)
    Vw = Vall[ks:p0 + n].numpy().reshape(-1, H, hd)
    o_ref, _ = O.swa(q.numpy().reshape(n, H, hd), Kw, Vw, qpos, kpos, window)
    cu = lambda t: t.to(tdt).cuda().contiguous()
    o = torch.empty(n, H * hd, device="cuda", dtype=tdt)
    lse = torch.empty(H, n, device="cuda")
    ops.swa_forward(cu(q), cu(kr), cu(vr), H, hd, p0, window, o, lse)
    ops.sync()
    err = np.abs(o.double().cpu().numpy().reshape(o_ref.shape) - o_ref).max()
    assert err <= 2e-2 * max(1.0, np.abs(o_ref).max()), err


def _normalised_case(H, hd, n, p0, window, ring, gq, gk, seed):
    """Queries and keys through an RMSNorm with gains gq, gk (the model's
    QK-norm), rounded to bf16; values plain normal."""
    Kall, Vall, q, _, _, _, tdt = _case(H, hd, n, p0, window, ring, "bf16", seed)

    def norm(x, g):
        x = x.view(x.shape[0], H, hd)
        y = x / torch.sqrt((x * x).mean(-1, keepdim=True) + 1e-5) * g
        return y.reshape(x.shape[0], H * hd).to(tdt).double()

    Kall, q = norm(Kall, gk), norm(q, gq)
    kr = torch.zeros(ring, H * hd, dtype=torch.float64)
    vr = torch.zeros(ring, H * hd, dtype=torch.float64)
    for j in range(p0 + n):
        kr[j % ring] = Kall[j]
        vr[j % ring] = Vall[j]
    return Kall, Vall, q, kr, vr, tdt


def _oracle_fwd(Kall, Vall, q, H, hd, n, p0, window):
    qpos = np.arange(p0, p0 + n)
    ks = max(0, p0 - window + 1)
    kpos = np.arange(ks, p0 + n)
    Kw = Kall[ks:p0 + n].numpy().reshape(-1, H, hd)
    Vw = Vall[ks:p0 + n].numpy().reshape(-1, H, hd)
    qq = q.numpy().reshape(n, H, hd)
    o_ref, _ = O.swa(qq, Kw, Vw, qpos, kpos, window)
    s = np.einsum("nhe,mhe->hnm", qq, Kw) / math.sqrt(hd)
    s = np.where(O.window_mask(qpos, kpos, window)[None], s, -np.inf)
    lse_ref = np.log(np.exp(s - s.max(-1, keepdims=True)).sum(-1)) + s.max(-1)
    return o_ref, lse_ref


FIXED_CASES = [(300, 1000, 700, 1152), (129, 0, 5000, 256), (200, 4000, 4096, 4352), (37, 5, 1, 64),
               (256, 1024, 1024, 2048)]
FIXED_VARIANTS = [(64, None), (80, 0), (80, 2), (80, 4), (96, None), (96, 4), (128, None), (128, 2)]


@pytest.mark.parametrize("hd,exp_poly", FIXED_VARIANTS)
@pytest.mark.parametrize("n,p0,window,ring", FIXED_CASES)
def test_tc_forward_fixed_shift_vs_oracle(hd, exp_poly, n, p0, window, ring):
    """Queries and keys of bounded norm (an RMSNorm with known gains): the
    fixed-shift forward (row shift from the norm bounds, part of 2^x from
    the FMA-pipe polynomial) against the oracle, and against the
    running-maximum forward of the same inputs."""
    from test_long_context_b200 import ops
    H = 2
    gen = torch.Generator().manual_seed(hd)
    gq = 0.5 + torch.rand(hd, generator=gen, dtype=torch.float64)
    gk = 0.5 + torch.rand(hd, generator=gen, dtype=torch.float64)
    Kall, Vall, q, kr, vr, tdt = _normalised_case(H, hd, n, p0, window, ring, gq, gk, seed=hd + n)
    o_ref, lse_ref = _oracle_fwd(Kall, Vall, q, H, hd, n, p0, window)
    cu = lambda t: t.to(tdt).cuda().contiguous()
    qd, krd, vrd = cu(q), cu(kr), cu(vr)
    bounds = dict(q_norm_max=float(gq.abs().max()) * hd ** 0.5, k_norm_max=float(gk.abs().max()) * hd ** 0.5)
    o = torch.empty(n, H * hd, device="cuda", dtype=tdt)
    lse = torch.empty(H, n, device="cuda")
    ops.swa_forward(qd, krd, vrd, H, hd, p0, window, o, lse, exp_poly=exp_poly, **bounds)
    o2 = torch.empty_like(o)
    lse2 = torch.empty_like(lse)
    ops.swa_forward(qd, krd, vrd, H, hd, p0, window, o2, lse2)  # running maximum
    ops.sync()
    om = max(1.0, np.abs(o_ref).max())
    assert np.abs(o.double().cpu().numpy().reshape(o_ref.shape) - o_ref).max() <= 2e-2 * om
    assert np.abs(lse.double().cpu().numpy() - lse_ref).max() <= 1e-3 * max(1.0, np.abs(lse_ref).max())
    # both round P to bf16, at different scales: a few bf16 steps of o apart at most
    assert (o.double() - o2.double()).abs().max().item() <= 2e-2 * om
    assert (lse - lse2).abs().max().item() <= 1e-3 * max(1.0, lse2.abs().max().item())


@pytest.mark.parametrize("hd", [80, 128])
def test_tc_forward_large_norm_bound_keeps_running_max(hd):
    """Norm bounds whose score bound exceeds 2^48 leave the fixed shift
    unused: the result is bit for bit the running-max forward's."""
    from test_long_context_b200 import ops
    H, n, p0, window, ring = 2, 200, 512, 300, 768
    g = torch.full((hd,), 6.0, dtype=torch.float64)
    Kall, Vall, q, kr, vr, tdt = _normalised_case(H, hd, n, p0, window, ring, g, g, seed=7)
    cu = lambda t: t.to(tdt).cuda().contiguous()
    o = torch.empty(n, H * hd, device="cuda", dtype=tdt)
    lse = torch.empty(H, n, device="cuda")
    b = 6.0 * hd ** 0.5
    ops.swa_forward(cu(q), cu(kr), cu(vr), H, hd, p0, window, o, lse, q_norm_max=b, k_norm_max=b)
    o2, lse2 = torch.empty_like(o), torch.empty_like(lse)
    ops.swa_forward(cu(q), cu(kr), cu(vr), H, hd, p0, window, o2, lse2)
    ops.sync()
    assert torch.equal(o, o2) and torch.equal(lse, lse2)
    o_ref, _ = _oracle_fwd(Kall, Vall, q, H, hd, n, p0, window)
    assert np.abs(o.double().cpu().numpy().reshape(o_ref.shape) - o_ref).max() <= 2e-2 * max(1.0, np.abs(o_ref).max())


@pytest.mark.parametrize("exp_poly", [0, 4])
def test_tc_forward_fixed_shift_tolerates_understated_key_bound(exp_poly):
    """Keys twice as long as the stated bound (inside the documented 3.5x),
    with keys planted equal to queries so that scores reach |q| |k|: the row
    shift is then below the largest score, P exceeds 1, and the result is
    still the oracle's."""
    from test_long_context_b200 import ops
    H, hd, n, p0, window, ring = 2, 80, 256, 1024, 1024, 2048
    g = torch.ones(hd, dtype=torch.float64)
    Kall, Vall, q, kr, vr, tdt = _normalised_case(H, hd, n, p0, window, ring, g, g, seed=9)
    for t, r in enumerate([3, 130, 200]):
        Kall[p0 + r - t] = q[r]
        kr[(p0 + r - t) % ring] = q[r]
    o_ref, lse_ref = _oracle_fwd(Kall, Vall, q, H, hd, n, p0, window)
    cu = lambda t: t.to(tdt).cuda().contiguous()
    o = torch.empty(n, H * hd, device="cuda", dtype=tdt)
    lse = torch.empty(H, n, device="cuda")
    ops.swa_forward(cu(q), cu(kr), cu(vr), H, hd, p0, window, o, lse, q_norm_max=hd ** 0.5,
                    k_norm_max=0.5 * hd ** 0.5, exp_poly=exp_poly)
    ops.sync()
    assert np.abs(o.double().cpu().numpy().reshape(o_ref.shape) - o_ref).max() <= 2e-2 * max(1.0, np.abs(o_ref).max())
    assert np.abs(lse.double().cpu().numpy() - lse_ref).max() <= 1e-3 * max(1.0, np.abs(lse_ref).max())


def test_watchdog_bounded_wait_reports_timeout():
    """A wait on a barrier nothing arrives at gives up and is reported as
    TTT_ERR_TIMEOUT; the device stays usable afterwards."""
    from test_long_context_b200 import _lib as L
    from test_long_context_b200 import ops
    ops.watchdog_selftest()
    with pytest.raises(L.TTTError) as e:
        ops.sync()
    assert e.value.code == L.TTT_ERR_TIMEOUT
    ops.sync()  # cleared; the context still works
    x = torch.ones(4, device="cuda")
    assert float(x.sum()) == 4.0
