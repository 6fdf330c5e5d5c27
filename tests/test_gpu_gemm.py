"""GEMM kernels through the op-level C ABI vs torch (fp64 reference of the
same rounded operands).  tcgen05 path for bf16, SIMT path for fp32."""
import pytest
import torch

pytestmark = pytest.mark.gpu

SHAPES = [(256, 512, 256), (200, 392, 136), (128, 128, 64), (1000, 1280, 520)]
COMBOS = [(0, 0), (0, 1), (1, 1)]


def _operands(M, N, K, a_mn, b_mn, dtype, seed=0):
    g = torch.Generator(device="cuda").manual_seed(seed)
    A = torch.randn((K, M) if a_mn else (M, K), device="cuda", generator=g).to(dtype)
    B = torch.randn((K, N) if b_mn else (N, K), device="cuda", generator=g).to(dtype)
    Am = A.double().T if a_mn else A.double()
    Bm = B.double() if b_mn else B.double().T
    return A, B, Am @ Bm  # [M, N]


@pytest.mark.parametrize("shape", SHAPES)
@pytest.mark.parametrize("combo", COMBOS)
@pytest.mark.parametrize("bn", [128, 256])
def test_tc_gemm_store(shape, combo, bn):
    from test_long_context_b200 import ops
    M, N, K = shape
    A, B, ref = _operands(M, N, K, *combo, torch.bfloat16)
    c = torch.full((M, N), float("nan"), device="cuda")
    ops.gemm(A, B, *combo, ops.L.EPI_STORE_F32, c=c, bn=bn)
    ops.sync()
    err = (c.double() - ref).abs().max().item()
    assert err <= 1e-4 * ref.abs().max().item() + 1e-4, err


@pytest.mark.parametrize("combo", COMBOS)
def test_simt_gemm_store(combo):
    from test_long_context_b200 import ops
    M, N, K = 200, 392, 136
    A, B, ref = _operands(M, N, K, *combo, torch.float32)
    c = torch.full((M, N), float("nan"), device="cuda")
    ops.gemm(A, B, *combo, ops.L.EPI_STORE_F32, c=c)
    ops.sync()
    assert (c.double() - ref).abs().max().item() <= 1e-4


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
def test_gemm_add_swiglu_sgd(dtype):
    from test_long_context_b200 import ops
    M, N, K = 300, 512, 192
    A, B, ref = _operands(M, N, K, 0, 0, dtype, seed=1)
    tol = 2e-2 if dtype == torch.bfloat16 else 1e-4
    # residual add
    x0 = torch.randn(M, N, device="cuda")
    x = x0.clone()
    ops.gemm(A, B, 0, 0, ops.L.EPI_ADD_F32, c=x)
    ops.sync()
    assert (x.double() - (x0.double() + ref)).abs().max().item() <= 1e-4 * ref.abs().max().item() + 1e-4
    # SwiGLU over (gate 64 | up 64) column pairs
    a = torch.empty(M, N // 2, device="cuda", dtype=dtype)
    raw = torch.empty(M, N, device="cuda", dtype=dtype)
    ops.gemm(A, B, 0, 0, ops.L.EPI_SWIGLU, c=a, c2=raw)
    ops.sync()
    r = ref.view(M, N // 128, 2, 64)
    g, u = r[:, :, 0], r[:, :, 1]
    want = (torch.nn.functional.silu(g) * u).reshape(M, N // 2)
    assert (a.double() - want).abs().max().item() <= tol * want.abs().max().item()
    assert (raw.double() - ref).abs().max().item() <= tol * ref.abs().max().item()
    # SGD epilogue on a weight-gradient-shaped product
    Aw, Bw, G = _operands(160, 384, 256, 1, 1, dtype, seed=2) if dtype == torch.bfloat16 else _operands(160, 384, 256, 1, 1, dtype, seed=2)
    W = torch.randn(160, 384, device="cuda")
    W0 = W.clone()
    W16 = torch.empty(160, 384, device="cuda", dtype=torch.bfloat16) if dtype == torch.bfloat16 else None
    ops.gemm(Aw, Bw, 1, 1, ops.L.EPI_SGD, c=W, c2=W16, alpha=0.01)
    ops.sync()
    want = W0.double() - 0.01 * G
    assert (W.double() - want).abs().max().item() <= 1e-5
    if W16 is not None:
        assert torch.equal(W16, W.to(torch.bfloat16))


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
def test_gemm_cross_entropy_epilogues(dtype):
    from test_long_context_b200 import ops
    M, V, K = 260, 1000, 128  # ragged rows and vocab
    h = (torch.randn(M, K, device="cuda") * 0.5).to(dtype)
    W = (torch.randn(V, K, device="cuda") * 0.5).to(dtype)
    z = h.double() @ W.double().T
    tgt = torch.randint(0, V, (M,), device="cuda", dtype=torch.int32)
    bf = dtype == torch.bfloat16
    nt = ops.gemm_ce_tiles(bf, M, V)
    pm = torch.empty(nt, M, device="cuda")
    ps = torch.empty(nt, M, device="cuda")
    zt = torch.full((M,), float("nan"), device="cuda")
    ops.gemm(h, W, 0, 0, ops.L.EPI_CE_FWD, row_i=tgt, part_max=pm, part_sum=ps, target_logit=zt, part_ld=M)
    ops.sync()
    gm = pm.max(0).values
    lse = gm + torch.log((ps * torch.exp(pm - gm)).sum(0))
    want_lse = torch.logsumexp(z, 1)
    assert (lse.double() - want_lse).abs().max().item() <= 1e-4
    assert (zt.double() - z.gather(1, tgt.long()[:, None])[:, 0]).abs().max().item() <= 1e-4
    # backward: dz = (softmax - onehot) * scale, columns offset by a vocab chunk start
    scale = torch.full((M,), 1.0 / M, device="cuda")
    scale[-3:] = 0
    off = 300
    dz = torch.empty(M, V - off, device="cuda", dtype=dtype)
    ops.gemm(h, W[off:], 0, 0, ops.L.EPI_CE_BWD, c=dz, row_f=want_lse.float(), row_g=scale, row_i=tgt,
             col_offset=off)
    ops.sync()
    p = torch.softmax(z, 1)
    oh = torch.nn.functional.one_hot(tgt.long(), V).double()
    want = ((p - oh) * scale.double()[:, None])[:, off:]
    assert (dz.double() - want).abs().max().item() <= (1e-2 if bf else 2e-5) * want.abs().max().item()


@pytest.mark.parametrize("combo", [(0, 0), (0, 1)])
@pytest.mark.parametrize("ksplit", [2, 3, 7])
def test_split_k_matches_and_is_deterministic(combo, ksplit):
    """Split-K partials summed in a fixed order: equal to the product within
    fp32 accumulation error, with every epilogue, and bit-identical on rerun."""
    from test_long_context_b200 import ops
    M, N, K = 300, 640, 4160   # ragged rows; K not a multiple of the split
    A, B, ref = _operands(M, N, K, *combo, torch.bfloat16, seed=9)
    ws = torch.empty(ksplit * M * N, device="cuda")
    c = torch.empty(M, N, device="cuda")
    ops.gemm_split(A, B, *combo, ops.L.EPI_STORE_F32, ksplit, ws, c=c)
    c_again = torch.empty_like(c)
    ops.gemm_split(A, B, *combo, ops.L.EPI_STORE_F32, ksplit, ws, c=c_again)
    x0 = torch.randn(M, N, device="cuda")
    x = torch.empty_like(x0)
    ops.gemm_split(A, B, *combo, ops.L.EPI_ADD_F32, ksplit, ws, c=x, c2=x0)
    cb = torch.empty(M, N, device="cuda", dtype=torch.bfloat16)
    ops.gemm_split(A, B, *combo, ops.L.EPI_STORE_BF16, ksplit, ws, c=cb)
    ops.sync()
    scale = ref.abs().max().item()
    assert (c.double() - ref).abs().max().item() <= 1e-4 * scale + 1e-4
    assert torch.equal(c, c_again)
    assert (x.double() - (x0.double() + ref)).abs().max().item() <= 1e-4 * scale + 1e-4
    assert (cb.double() - ref).abs().max().item() <= 1e-2 * scale


def _dual_ref(A, B, A2, B2, a_mn, b_mn, n_ext):
    Am = A.double().T if a_mn else A.double()
    Bm = B.double() if b_mn else B.double().T
    A2m = A2.double().T if a_mn else A2.double()
    B2m = B2.double() if b_mn else B2.double().T
    ref = Am @ Bm
    ref[:, n_ext:] += A2m @ B2m
    return ref


@pytest.mark.parametrize("combo", [(0, 0), (0, 1)])
def test_dual_product_swiglu_mixed_tiles(combo):
    """Second product on the columns from n_ext on only (the fast half of a
    [static | fast] gate/up GEMM), a different reduction length K2."""
    from test_long_context_b200 import ops
    M, N, K, K2, n_ext = 300, 768, 192, 136, 384
    g = torch.Generator(device="cuda").manual_seed(21)
    a_mn, b_mn = combo
    A = torch.randn((M, K), device="cuda", generator=g).bfloat16()
    B = torch.randn((K, N) if b_mn else (N, K), device="cuda", generator=g).bfloat16()
    A2 = torch.randn((M, K2), device="cuda", generator=g).bfloat16()
    B2 = torch.randn((K2, N - n_ext) if b_mn else (N - n_ext, K2), device="cuda", generator=g).bfloat16()
    ref = _dual_ref(A, B, A2, B2, a_mn, b_mn, n_ext)
    a = torch.empty(M, N // 2, device="cuda", dtype=torch.bfloat16)
    raw = torch.empty(M, N, device="cuda", dtype=torch.bfloat16)
    ops.gemm_dual(A, B, A2, B2, a_mn, b_mn, ops.L.EPI_SWIGLU, n_ext=n_ext, bn=128, c=a, c2=raw)
    c = torch.full((M, N), float("nan"), device="cuda")
    ops.gemm_dual(A, B, A2, B2, a_mn, b_mn, ops.L.EPI_STORE_F32, n_ext=n_ext, bn=128, c=c)
    ops.sync()
    assert (c.double() - ref).abs().max().item() <= 1e-4 * ref.abs().max().item() + 1e-4
    r = ref.view(M, N // 128, 2, 64)
    want = (torch.nn.functional.silu(r[:, :, 0]) * r[:, :, 1]).reshape(M, N // 2)
    assert (a.double() - want).abs().max().item() <= 2e-2 * want.abs().max().item()
    assert (raw.double() - ref).abs().max().item() <= 2e-2 * ref.abs().max().item()


@pytest.mark.parametrize("ksplit", [1, 3, 5])
def test_dual_product_add_split_k(ksplit):
    """Second product on every tile with split-K over the concatenated
    reduction: ragged K (a partial last k-block before the second product
    starts) and ragged K2; deterministic on rerun."""
    from test_long_context_b200 import ops
    M, N, K, K2 = 300, 640, 4104, 1000
    g = torch.Generator(device="cuda").manual_seed(22)
    A = torch.randn((M, K), device="cuda", generator=g).bfloat16()
    B = torch.randn((N, K), device="cuda", generator=g).bfloat16()
    A2 = torch.randn((M, K2), device="cuda", generator=g).bfloat16()
    B2 = torch.randn((N, K2), device="cuda", generator=g).bfloat16()
    ref = _dual_ref(A, B, A2, B2, 0, 0, 0)
    ws = torch.empty(max(ksplit, 1) * M * N, device="cuda")
    x0 = torch.randn(M, N, device="cuda")
    x, x_again = torch.empty_like(x0), torch.empty_like(x0)
    ops.gemm_dual(A, B, A2, B2, 0, 0, ops.L.EPI_ADD_F32, ksplit=ksplit, workspace=ws, c=x, c2=x0)
    ops.gemm_dual(A, B, A2, B2, 0, 0, ops.L.EPI_ADD_F32, ksplit=ksplit, workspace=ws, c=x_again, c2=x0)
    ops.sync()
    assert (x.double() - (x0.double() + ref)).abs().max().item() <= 1e-4 * ref.abs().max().item() + 1e-4
    assert torch.equal(x, x_again)


def test_sgd_two_term_bf16_shadow():
    """SGD epilogue with hi and lo shadows: hi = bf16(W), lo = bf16(W - hi),
    so hi + lo follows an update far below one bf16 ulp of W."""
    from test_long_context_b200 import ops
    Aw, Bw, G = _operands(160, 384, 256, 1, 1, torch.bfloat16, seed=3)
    W = (0.02 * torch.randn(160, 384, device="cuda")).bfloat16().float()  # weight-sized, bf16-exact start
    W0 = W.clone()
    hi = torch.empty(160, 384, device="cuda", dtype=torch.bfloat16)
    lo = torch.empty_like(hi)
    alpha = 1e-6
    ops.gemm(Aw, Bw, 1, 1, ops.L.EPI_SGD, c=W, c2=hi, c3=lo, alpha=alpha)
    ops.sync()
    want = W0.double() - alpha * G
    assert (W.double() - want).abs().max().item() <= 1e-6
    assert torch.equal(hi, W.to(torch.bfloat16))
    assert torch.equal(lo, (W - hi.float()).to(torch.bfloat16))
    two = hi.double() + lo.double()
    step = (want - W0.double()).abs()
    # hi + lo carries W to ~|W| 2^-18, well inside 1% of the largest step
    assert (two - want).abs().max().item() <= 1e-2 * step.max().item()
    # a single bf16 copy would lose most of the step (half an ulp of 0.02 is ~6e-5)
    assert (hi.double() - W0.double()).abs().mean().item() < 0.5 * step.mean().item()


def test_read_modify_write_epilogues_many_tiles():
    """SGD (hi + lo shadows) and residual-add epilogues on shapes with more
    work units than SMs (each persistent CTA drains several tiles in both
    epilogue groups), ragged rows and a last n-tile that is only partly
    inside N, so the read-ahead of the master / residual meets every edge."""
    from test_long_context_b200 import ops
    M, N, K = 2600, 2600, 192
    Aw, Bw, G = _operands(M, N, K, 1, 1, torch.bfloat16, seed=5)
    W = 0.02 * torch.randn(M, N, device="cuda")
    W0 = W.clone()
    hi = torch.full((M, N), float("nan"), device="cuda", dtype=torch.bfloat16)
    lo = torch.full_like(hi, float("nan"))
    ops.gemm(Aw, Bw, 1, 1, ops.L.EPI_SGD, c=W, c2=hi, c3=lo, alpha=1e-3)
    ops.sync()
    assert (W.double() - (W0.double() - 1e-3 * G)).abs().max().item() <= 1e-6
    assert torch.equal(hi, W.to(torch.bfloat16))
    assert torch.equal(lo, (W - hi.float()).to(torch.bfloat16))
    # residual add into a separate output (c2 = residual), K-major operands
    A, B, ref = _operands(M, N, K, 0, 0, torch.bfloat16, seed=6)
    x0 = torch.randn(M, N, device="cuda")
    x = torch.full((M, N), float("nan"), device="cuda")
    ops.gemm(A, B, 0, 0, ops.L.EPI_ADD_F32, c=x, c2=x0)
    ops.sync()
    assert (x.double() - (x0.double() + ref)).abs().max().item() <= 1e-4 * ref.abs().max().item() + 1e-4


@pytest.mark.parametrize("N", [2600, 2602])
def test_split_k_reduce_vector_and_scalar_paths(N):
    """The ordered split-K sum reads float4 when a row's 4 columns are
    16-byte aligned (N % 4 == 0) and falls back to scalars otherwise; both
    give the same in-order sum."""
    from test_long_context_b200 import ops
    M, K, S = 260, 4096, 4
    A, B, ref = _operands(M, N, K, 0, 0, torch.bfloat16, seed=7)
    ws = torch.empty(S * M * N, device="cuda")
    x0 = torch.randn(M, N, device="cuda")
    x = x0.clone()
    ops.gemm_split(A, B, 0, 0, ops.L.EPI_ADD_F32, S, ws, c=x)
    c = torch.full((M, N), float("nan"), device="cuda")
    ops.gemm_split(A, B, 0, 0, ops.L.EPI_STORE_F32, S, ws, c=c)
    ops.sync()
    tol = 1e-4 * ref.abs().max().item() + 1e-4
    assert (c.double() - ref).abs().max().item() <= tol
    assert (x.double() - (x0.double() + ref)).abs().max().item() <= tol


@pytest.mark.parametrize("combo", COMBOS)
def test_cta_pair_tiles_every_epilogue(combo):
    """GEMMs with more than 128 rows run on CTA pairs (one 256 x BN tile per
    pair, each CTA loading its own 128 rows of A and half of the B tile):
    every epilogue on 128- and 256-wide pair tiles against the fp64 product
    and against each other, with a last pair tile whose odd CTA has no valid
    rows at all (M = 600)."""
    from test_long_context_b200 import ops
    M, N, K = 600, 768, 320
    A, B, ref = _operands(M, N, K, *combo, torch.bfloat16, seed=31)
    scale = ref.abs().max().item()
    outs = {}
    for bn in (128, 256):
        c = torch.full((M, N), float("nan"), device="cuda")
        ops.gemm(A, B, *combo, ops.L.EPI_STORE_F32, c=c, bn=bn)
        cb = torch.full((M, N), float("nan"), device="cuda", dtype=torch.bfloat16)
        ops.gemm(A, B, *combo, ops.L.EPI_STORE_BF16, c=cb, bn=bn)
        x0 = torch.randn(M, N, device="cuda", generator=torch.Generator(device="cuda").manual_seed(1))
        x = torch.full_like(x0, float("nan"))
        ops.gemm(A, B, *combo, ops.L.EPI_ADD_F32, c=x, c2=x0, bn=bn)
        a = torch.full((M, N // 2), float("nan"), device="cuda", dtype=torch.bfloat16)
        raw = torch.full((M, N), float("nan"), device="cuda", dtype=torch.bfloat16)
        ops.gemm(A, B, *combo, ops.L.EPI_SWIGLU, c=a, c2=raw, bn=bn)
        W = (0.02 * torch.randn(M, N, device="cuda", generator=torch.Generator(device="cuda").manual_seed(2)))
        W0 = W.clone()
        hi = torch.full((M, N), float("nan"), device="cuda", dtype=torch.bfloat16)
        lo = torch.full_like(hi, float("nan"))
        ops.gemm(A, B, *combo, ops.L.EPI_SGD, c=W, c2=hi, c3=lo, alpha=1e-3, bn=bn)
        ops.sync()
        assert (c.double() - ref).abs().max().item() <= 1e-4 * scale + 1e-4, bn
        assert (cb.double() - ref).abs().max().item() <= 1e-2 * scale, bn
        assert (x.double() - (x0.double() + ref)).abs().max().item() <= 1e-4 * scale + 1e-4, bn
        r = ref.view(M, N // 128, 2, 64)
        want = (torch.nn.functional.silu(r[:, :, 0]) * r[:, :, 1]).reshape(M, N // 2)
        assert (a.double() - want).abs().max().item() <= 2e-2 * want.abs().max().item(), bn
        assert (W.double() - (W0.double() - 1e-3 * ref)).abs().max().item() <= 1e-6 * scale + 1e-6, bn
        assert torch.equal(hi, W.to(torch.bfloat16)) and torch.equal(lo, (W - hi.float()).to(torch.bfloat16))
        outs[bn] = c
    assert (outs[128] - outs[256]).abs().max().item() <= 1e-5 * scale


def test_cta_pair_tiles_cross_entropy_split_and_dual():
    """CE partials / CE gradient, split-K partials and a second product on
    256-wide pair tiles."""
    from test_long_context_b200 import ops
    M, V, K = 520, 1000, 192
    h = (torch.randn(M, K, device="cuda") * 0.5).bfloat16()
    W = (torch.randn(V, K, device="cuda") * 0.5).bfloat16()
    z = h.double() @ W.double().T
    tgt = torch.randint(0, V, (M,), device="cuda", dtype=torch.int32)
    nt = ops.gemm_ce_tiles(True, M, V, 256)
    pm, ps = torch.empty(nt, M, device="cuda"), torch.empty(nt, M, device="cuda")
    zt = torch.full((M,), float("nan"), device="cuda")
    logits = torch.full((M, V), float("nan"), device="cuda")
    ops.gemm(h, W, 0, 0, ops.L.EPI_CE_FWD, c=logits, row_i=tgt, part_max=pm, part_sum=ps, target_logit=zt,
             part_ld=M, bn=256)
    plain = torch.full((M, V), float("nan"), device="cuda")
    ops.gemm(h, W, 0, 0, ops.L.EPI_STORE_F32, c=plain, bn=256)
    want_lse = torch.logsumexp(z, 1)
    dz = torch.empty(M, V, device="cuda", dtype=torch.bfloat16)
    scale = torch.full((M,), 1.0 / M, device="cuda")
    ops.gemm(h, W, 0, 0, ops.L.EPI_CE_BWD, c=dz, row_f=want_lse.float(), row_g=scale, row_i=tgt, bn=256)
    ops.sync()
    gm = pm.max(0).values
    lse = gm + torch.log((ps * torch.exp(pm - gm)).sum(0))
    assert (lse.double() - want_lse).abs().max().item() <= 1e-4
    assert (zt.double() - z.gather(1, tgt.long()[:, None])[:, 0]).abs().max().item() <= 1e-4
    # the kept logits are the accumulator itself: the plain product's values, bit for bit
    assert torch.equal(logits, plain)
    p = torch.softmax(z, 1)
    oh = torch.nn.functional.one_hot(tgt.long(), V).double()
    want = (p - oh) * scale.double()[:, None]
    assert (dz.double() - want).abs().max().item() <= 1e-2 * want.abs().max().item()
    # split-K partials on pair tiles, then the ordered sum
    Ms, Ns, Ks, S = 300, 640, 4160, 3
    A, B, ref = _operands(Ms, Ns, Ks, 0, 0, torch.bfloat16, seed=33)
    ws = torch.empty(S * Ms * Ns, device="cuda")
    c = torch.full((Ms, Ns), float("nan"), device="cuda")
    ops.gemm_split(A, B, 0, 0, ops.L.EPI_STORE_F32, S, ws, c=c, bn=256)
    # second product on the columns from n_ext on (a multiple of the 256-wide tile)
    Md, Nd, Kd, K2, n_ext = 300, 1024, 192, 136, 512
    g = torch.Generator(device="cuda").manual_seed(34)
    Ad = torch.randn((Md, Kd), device="cuda", generator=g).bfloat16()
    Bd = torch.randn((Nd, Kd), device="cuda", generator=g).bfloat16()
    A2 = torch.randn((Md, K2), device="cuda", generator=g).bfloat16()
    B2 = torch.randn((Nd - n_ext, K2), device="cuda", generator=g).bfloat16()
    refd = _dual_ref(Ad, Bd, A2, B2, 0, 0, n_ext)
    cd = torch.full((Md, Nd), float("nan"), device="cuda")
    ops.gemm_dual(Ad, Bd, A2, B2, 0, 0, ops.L.EPI_STORE_F32, n_ext=n_ext, bn=256, c=cd)
    ops.sync()
    assert (c.double() - ref).abs().max().item() <= 1e-4 * ref.abs().max().item() + 1e-4
    assert (cd.double() - refd).abs().max().item() <= 1e-4 * refd.abs().max().item() + 1e-4


@pytest.mark.parametrize("combo", [(0, 0), (0, 1), (1, 1)])
def test_pair_tiles_160_wide(combo):
    """160-wide pair tiles (the M = b products of the prefill: a single wave
    of 256 x 160 tiles): plain stores, the residual add and split-K partials
    against the fp64 product, on a ragged N (1000: the last tile holds 40
    columns) and a last pair tile whose odd CTA has no rows (M = 600)."""
    from test_long_context_b200 import ops
    M, N, K = 600, 1000, 704
    A, B, ref = _operands(M, N, K, *combo, torch.bfloat16, seed=37)
    scale = ref.abs().max().item()
    c = torch.full((M, N), float("nan"), device="cuda")
    ops.gemm(A, B, *combo, ops.L.EPI_STORE_F32, c=c, bn=160)
    cb = torch.full((M, N), float("nan"), device="cuda", dtype=torch.bfloat16)
    ops.gemm(A, B, *combo, ops.L.EPI_STORE_BF16, c=cb, bn=160)
    x0 = torch.randn(M, N, device="cuda", generator=torch.Generator(device="cuda").manual_seed(3))
    x = torch.full_like(x0, float("nan"))
    ops.gemm(A, B, *combo, ops.L.EPI_ADD_F32, c=x, c2=x0, bn=160)
    ws = torch.empty(3 * M * N, device="cuda")
    cs = torch.full((M, N), float("nan"), device="cuda")
    ops.gemm_split(A, B, *combo, ops.L.EPI_STORE_F32, 3, ws, c=cs, bn=160)
    c128 = torch.full((M, N), float("nan"), device="cuda")
    ops.gemm(A, B, *combo, ops.L.EPI_STORE_F32, c=c128, bn=128)
    ops.sync()
    assert (c.double() - ref).abs().max().item() <= 1e-4 * scale + 1e-4
    assert (cb.double() - ref).abs().max().item() <= 1e-2 * scale
    assert (x.double() - (x0.double() + ref)).abs().max().item() <= 1e-4 * scale + 1e-4
    assert (cs.double() - ref).abs().max().item() <= 1e-4 * scale + 1e-4
    assert (c - c128).abs().max().item() <= 1e-5 * scale


def test_pair_tiles_160_wide_refused_where_unsupported():
    """160-wide tiles are refused for epilogues that need 128-column groups
    (SwiGLU, CE, SGD) and for single-CTA products (M <= 128)."""
    from test_long_context_b200 import _lib as L
    from test_long_context_b200 import ops
    A = torch.randn(600, 256, device="cuda").bfloat16()
    B = torch.randn(512, 256, device="cuda").bfloat16()
    a = torch.empty(600, 256, device="cuda", dtype=torch.bfloat16)
    with pytest.raises(L.TTTError):
        ops.gemm(A, B, 0, 0, ops.L.EPI_SWIGLU, c=a, bn=160)
    c = torch.empty(100, 512, device="cuda")
    with pytest.raises(L.TTTError):
        ops.gemm(A[:100], B, 0, 0, ops.L.EPI_STORE_F32, c=c, bn=160)


def test_gemm_plan_of_the_prefill_products():
    """The plan picks one wave of 160-wide pair tiles for the b x d outputs
    of the blocks with fast weights, and 256-wide tiles for the large ones."""
    from test_long_context_b200 import ops
    S, bn = ops.gemm_plan(1024, 2560, 2560, ops.L.EPI_ADD_F32)
    assert (S, bn) == (1, 160)
    S, bn = ops.gemm_plan(16384, 2560, 2560, ops.L.EPI_ADD_F32)
    assert (S, bn) == (1, 256)
    S, bn = ops.gemm_plan(1024, 2560, 2560, ops.L.EPI_SWIGLU)
    assert (S, bn) == (1, 0)


def test_grouped_raster_large_operands():
    """A and B both larger than a third of L2 (here 52 MB each): the tiles
    are walked in groups of m-tiles (m fastest inside a group, one n-tile
    after the other).  Every output row block and column block is checked
    against the fp64 product, with the plain store and with SwiGLU."""
    from test_long_context_b200 import ops
    M, N, K = 12800, 12800, 2048
    g = torch.Generator(device="cuda").manual_seed(41)
    A = torch.randn(M, K, device="cuda", generator=g).to(torch.bfloat16)
    B = torch.randn(N, K, device="cuda", generator=g).to(torch.bfloat16)
    c = torch.full((M, N), float("nan"), device="cuda")
    ops.gemm(A, B, 0, 0, ops.L.EPI_STORE_F32, c=c)
    a = torch.full((M, N // 2), float("nan"), device="cuda", dtype=torch.bfloat16)
    ops.gemm(A, B, 0, 0, ops.L.EPI_SWIGLU, c=a)
    ops.sync()
    Bd = B.double()
    for r0 in range(0, M, 1600):  # one 128-row block per group-sized stride, every column
        rows = slice(r0, r0 + 128)
        ref = A[rows].double() @ Bd.T
        scale = ref.abs().max().item()
        assert (c[rows].double() - ref).abs().max().item() <= 1e-4 * scale + 1e-4, r0
        r = ref.view(128, N // 128, 2, 64)
        want = (torch.nn.functional.silu(r[:, :, 0]) * r[:, :, 1]).reshape(128, N // 2)
        assert (a[rows].double() - want).abs().max().item() <= 2e-2 * want.abs().max().item(), r0
    assert not torch.isnan(c).any() and not torch.isnan(a.float()).any()
