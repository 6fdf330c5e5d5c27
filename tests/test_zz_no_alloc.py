"""The allocation-free attention backward (ttt_op_swa_backward_noalloc),
for callers that may not allocate device memory, against the entry point
that takes caller scratch.  Collected last on purpose: if it fails, a run that
stops at the first failure has already run every other test."""
import ctypes

import pytest
import torch

pytestmark = pytest.mark.gpu


def _inputs(H, hd, n, p0, window, ring, dtype, seed):
    g = torch.Generator(device="cuda").manual_seed(seed)
    mk = lambda *s: torch.randn(*s, device="cuda", generator=g).to(dtype)
    return mk(n, H * hd), mk(ring, H * hd), mk(ring, H * hd), mk(n, H * hd)


@pytest.mark.parametrize("force_simt", [False, True])
@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
def test_noalloc_backward_matches_scratch_entry_point_twice(dtype, force_simt):
    """The allocation-free call runs the kernels that ttt_op_swa_backward runs
    with default flags (tensor cores for bf16 with head_dim 64, a ring of
    whole 128-row tiles; dk/dv on tensor cores when the chunk starts a tile),
    so against that call it must agree within the test tolerance; against the
    forced-SIMT call it agrees within bf16 rounding."""
    from test_long_context_b200 import ops
    H, hd, window, ring = 4, 64, 300, 512
    # two calls in a row with different shapes and inputs: the shared work
    # array must not carry anything from one call into the next; the second
    # call starts on a 128-row tile, so bf16 takes the tensor-core dk/dv kernel
    for call, (n, p0, seed) in enumerate([(200, 250, 1), (128, 384, 2)]):
        q, kr, vr, dout = _inputs(H, hd, n, p0, window, ring, dtype, seed)
        o = torch.empty_like(q)
        lse = torch.empty(H, n, device="cuda")
        ops.swa_forward(q, kr, vr, H, hd, p0, window, o, lse, force_simt=True)
        ref = [torch.empty_like(q) for _ in range(3)]
        D = torch.empty(H * n, device="cuda")
        ops.swa_backward(q, kr, vr, H, hd, p0, window, o, lse, dout, *ref, D, force_simt=force_simt)
        got = [torch.full_like(q, float("nan")) for _ in range(3)]
        ops.swa_backward_noalloc(q, kr, vr, H, hd, p0, window, o, lse, dout, *got)
        ops.sync()
        tol = 2e-2 if dtype == torch.bfloat16 else 1e-5
        for name, a, b in zip(("dq", "dk", "dv"), got, ref):
            err = (a.float() - b.float()).abs().max().item()
            assert err <= tol * max(1.0, b.float().abs().max().item()), (call, name, err)
            if not force_simt:
                assert torch.equal(a, b), (call, name, "same kernels, same inputs: results must be identical")


def test_noalloc_rejects_sizes_beyond_the_work_array():
    from test_long_context_b200 import _lib as L
    from test_long_context_b200 import ops
    H, hd = 64, 64
    n = (1 << 18) // H + 1          # n_heads * n_q just over the 262144-row limit
    q = torch.zeros(n, H * hd, device="cuda", dtype=torch.bfloat16)
    kr = torch.zeros(128, H * hd, device="cuda", dtype=torch.bfloat16)
    lse = torch.zeros(H, n, device="cuda")
    with pytest.raises(L.TTTError) as e:
        ops.swa_backward_noalloc(q, kr, kr, H, hd, 0, 4, q, lse, q, q, q, q)
    assert e.value.code == L.TTT_ERR_INVALID_ARG
    assert "262144" in str(e.value)
