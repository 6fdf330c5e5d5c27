"""Memory-bound kernels through their op-level entry points (ttt_ops.h)
against plain PyTorch / the oracle's formulas, at ragged sizes: RMSNorm,
QK-norm + RoPE with the ring write, SwiGLU backward, the generation
matrix-vector product with each epilogue, and single-query attention."""
import math

import numpy as np
import pytest
import torch

from oracle import ttt_oracle as O

pytestmark = pytest.mark.gpu

bf = torch.bfloat16


def test_rmsnorm():
    from test_long_context_b200 import ops
    g = torch.Generator(device="cuda").manual_seed(0)
    n, d = 37, 2560
    x = torch.randn(n, d, device="cuda", generator=g) * 3
    gain = 1 + 0.3 * torch.randn(d, device="cuda", generator=g)
    y = torch.empty(n, d, device="cuda", dtype=bf)
    r = torch.empty(n, device="cuda")
    ops.rmsnorm(x, gain, 1e-5, y, r)
    ops.sync()
    rr = torch.rsqrt((x.double() ** 2).mean(1) + 1e-5)
    assert torch.allclose(r.double(), rr, rtol=1e-5)
    want = (x.double() * rr[:, None] * gain.double())
    assert (y.double() - want).abs().max().item() <= 8e-3 * want.abs().max().item()


@pytest.mark.parametrize("hd", [64, 80, 128])
def test_qknorm_rope_and_ring_write(hd):
    from test_long_context_b200 import ops
    H, n, p0, R = 3, 45, 1000, 128
    d = H * hd
    gen = torch.Generator(device="cuda").manual_seed(hd)
    qkv = torch.randn(n, 3 * d, device="cuda", generator=gen).to(bf)
    gq = 1 + 0.3 * torch.randn(hd, device="cuda", generator=gen)
    gk = 1 + 0.3 * torch.randn(hd, device="cuda", generator=gen)
    qout = torch.empty(n, d, device="cuda", dtype=bf)
    kr = torch.zeros(R, d, device="cuda", dtype=bf)
    vr = torch.zeros(R, d, device="cuda", dtype=bf)
    rq = torch.empty(n, H, device="cuda")
    rk = torch.empty(n, H, device="cuda")
    tab = torch.empty(n * hd // 2 * 2, device="cuda")
    ops.qknorm_rope(qkv, p0, H, hd, 1e-5, 10000.0, gq, gk, qout, kr, vr, rq, rk, tab)
    ops.sync()
    a = qkv.double().cpu().numpy()
    pos = np.arange(p0, p0 + n)
    cos, sin = O.rope_tables(pos, hd, 10000.0)
    q = O.rope(O.rmsnorm(a[:, :d].reshape(n, H, hd), gq.double().cpu().numpy(), 1e-5)[0], cos, sin)
    k = O.rope(O.rmsnorm(a[:, d:2 * d].reshape(n, H, hd), gk.double().cpu().numpy(), 1e-5)[0], cos, sin)
    slots = pos % R
    assert np.abs(qout.double().cpu().numpy() - q.reshape(n, d)).max() <= 2e-2
    assert np.abs(kr.double().cpu().numpy()[slots] - k.reshape(n, d)).max() <= 2e-2
    assert np.array_equal(vr.cpu()[slots].view(torch.int16).numpy(), qkv[:, 2 * d:].cpu().view(torch.int16).numpy())


def test_swiglu_bwd():
    from test_long_context_b200 import ops
    gen = torch.Generator(device="cuda").manual_seed(3)
    n, F = 33, 384
    da = torch.randn(n, F, device="cuda", generator=gen).to(bf)
    gu = torch.randn(n, 2 * F, device="cuda", generator=gen).to(bf)
    dgu = torch.empty(n, 2 * F, device="cuda", dtype=bf)
    ops.swiglu_bwd(da, gu, dgu)
    ops.sync()
    r = gu.double().view(n, F // 64, 2, 64)
    gg, uu = r[:, :, 0], r[:, :, 1]
    s = torch.sigmoid(gg)
    dA = da.double().view(n, F // 64, 64)
    want = torch.stack([dA * uu * s * (1 + gg * (1 - s)), dA * gg * s], 2).reshape(n, 2 * F)
    assert (dgu.double() - want).abs().max().item() <= 1e-2 * want.abs().max().item()


@pytest.mark.parametrize("n,k", [(7680, 2560), (2560, 13824), (1000, 136)])
def test_gemv_epilogues(n, k):
    from test_long_context_b200 import ops
    gen = torch.Generator(device="cuda").manual_seed(n)
    W = (0.02 * torch.randn(n, k, device="cuda", generator=gen)).to(bf)
    x = torch.randn(k, device="cuda", generator=gen).to(bf)
    y = W.double() @ x.double()
    tol = 2e-5 * (W.double().abs() @ x.double().abs()).max().item() + 1e-6
    out = torch.empty(n, device="cuda", dtype=bf)
    ops.gemv(0, W, x, out)
    res = torch.randn(n, device="cuda", generator=gen)
    out2 = torch.empty(n, device="cuda")
    ops.gemv(1, W, x, out2, res=res)
    part = torch.empty(3 * 1184, device="cuda")
    tok = torch.empty(1, device="cuda", dtype=torch.int32)
    lse = torch.empty(1, device="cuda")
    ops.gemv(3, W, x, tok, lse=lse, part=part)
    ops.sync()
    assert (out.double() - y).abs().max().item() <= 1e-2 * y.abs().max().item() + tol
    assert (out2.double() - (res.double() + y)).abs().max().item() <= tol
    assert int(tok.item()) == int(torch.argmax(y).item())
    assert abs(lse.item() - torch.logsumexp(y, 0).item()) <= 1e-4
    if n % 128 == 0:
        a = torch.empty(n // 2, device="cuda", dtype=bf)
        raw = torch.empty(n, device="cuda", dtype=bf)
        ops.gemv(2, W, x, a, raw=raw)
        ops.sync()
        r = y.view(n // 128, 2, 64)
        want = (torch.nn.functional.silu(r[:, 0]) * r[:, 1]).reshape(n // 2)
        assert (a.double() - want).abs().max().item() <= 1e-2 * want.abs().max().item() + tol
        assert (raw.double() - y).abs().max().item() <= 1e-2 * y.abs().max().item() + tol


def test_gemv_greedy_ties_to_the_lowest_row():
    from test_long_context_b200 import ops
    n, k = 5000, 64
    W = torch.zeros(n, k, device="cuda", dtype=bf)
    W[[4321, 77, 2500], 0] = 1.0  # three rows tie for the maximum
    x = torch.zeros(k, device="cuda", dtype=bf)
    x[0] = 2.0
    part = torch.empty(3 * 1184, device="cuda")
    tok = torch.empty(1, device="cuda", dtype=torch.int32)
    lse = torch.empty(1, device="cuda")
    ops.gemv(3, W, x, tok, lse=lse, part=part)
    ops.sync()
    assert int(tok.item()) == 77
    want = math.log(3 * math.exp(2.0) + (n - 3))
    assert abs(lse.item() - want) <= 1e-4


@pytest.mark.parametrize("hd,p,window,R", [(80, 9000, 8192, 8320), (64, 100, 300, 512), (128, 700, 130, 256),
                                            (32, 0, 50, 64)])
def test_attn_decode(hd, p, window, R):
    from test_long_context_b200 import ops
    H = 3
    d = H * hd
    gen = torch.Generator(device="cuda").manual_seed(p)
    q = torch.randn(d, device="cuda", generator=gen).to(bf)
    kr = torch.randn(R, d, device="cuda", generator=gen).to(bf)
    vr = torch.randn(R, d, device="cuda", generator=gen).to(bf)
    o = torch.empty(d, device="cuda", dtype=bf)
    lse = torch.empty(H, device="cuda")
    # the last H words count finished splits: zero before the first call, left zero by every call
    ws = torch.zeros(H * (((window + 127) // 128 + 1) * (hd + 2) + 1), device="cuda")
    ops.attn_decode(q, kr, vr, H, hd, p, window, o, lse, ws)
    o2 = torch.empty_like(o)
    ops.attn_decode(q, kr, vr, H, hd, p, window, o2, None, ws)  # a second call on the same work space
    ops.sync()
    assert torch.equal(o, o2)
    assert (ws[-H:] == 0).all()
    lo = max(0, p - window + 1)
    pos = np.arange(lo, p + 1)
    K = kr.double().cpu().numpy()[pos % R].reshape(-1, H, hd)
    V = vr.double().cpu().numpy()[pos % R].reshape(-1, H, hd)
    qq = q.double().cpu().numpy().reshape(1, H, hd)
    want, P = O.swa(qq, K, V, np.array([p]), pos, window)
    s = np.einsum("nhe,mhe->hnm", qq, K) / math.sqrt(hd)
    lse_want = np.log(np.exp(s - s.max(-1, keepdims=True)).sum(-1)) + s.max(-1)
    assert np.abs(o.double().cpu().numpy() - want.reshape(d)).max() <= 1e-2
    assert np.abs(lse.double().cpu().numpy() - lse_want[:, 0]).max() <= 1e-4
