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
