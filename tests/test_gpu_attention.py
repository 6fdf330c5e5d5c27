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


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("hd", [32, 64, 80, 96])
@pytest.mark.parametrize("n,p0,window,ring", [(100, 350, 120, 256), (64, 0, 1000, 64), (37, 5, 1, 64),
                                              (130, 900, 64, 200)])
def test_swa_forward_backward_vs_oracle(dtype, hd, n, p0, window, ring):
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
    ops.swa_forward(qd, krd, vrd, H, hd, p0, window, o, lse)
    dq = torch.empty_like(o)
    dk = torch.empty_like(o)
    dv = torch.empty_like(o)
    D = torch.empty(H * n, device="cuda")
    ops.swa_backward(qd, krd, vrd, H, hd, p0, window, o, lse, dd, dq, dk, dv, D)
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
