"""Time single kernels of the prefill loop and of generation at a workload's shapes.

    python -m test_long_context_b200.opbench [--config 2.7b] [--op NAME ...] [--iters N]

Each op runs through the op-level C ABI (include/ttt_ops.h) on random
inputs of the exact shapes the engine uses for the named config, timed
with CUDA events after warm-up; one JSON line per op with the average
launch time and the algorithmic TFLOP/s (contractions) or GB/s (the
memory-bound kernels: algorithmic bytes = every operand read and every
result written once).  Only the requested ops get inputs, so with one --op,
--iters 1 --warmup 0 it is also the small, self-contained command that ncu
captures (one op's buffers on the device, nothing else launched).
"""
from __future__ import annotations

import argparse
import json
import os
import sys

import torch

sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))

from synth import get_config  # noqa: E402
from test_long_context_b200 import _lib as L  # noqa: E402
from test_long_context_b200 import ops  # noqa: E402


def band_pairs(p0, n, k):
    s = 0
    for p in range(p0, p0 + n):
        s += min(p + 1, k)
    return s


def meta_grad_flops(n_chunks, b, d, f, V):
    """GEMM flops of ttt_op_meta_grad: the inner loop runs every chunk's
    forward and backward (9 products: 7 of b x d x f, 2 of b x d x V); the
    reverse sweep runs them again for chunks N-2 .. 0 plus their tangents (14
    products: 10 of b x d x f, 2 of b x d x V)."""
    fb = 2.0 * b * (7 * d * f + 2 * d * V)
    hv = 2.0 * b * (10 * d * f + 2 * d * V)
    return n_chunks * fb + (n_chunks - 1) * (fb + hv)


def meta_grad_inputs(n_chunks, b, d, f, V, seed=0):
    """Seeded synthetic inputs of the meta-gradient at a model's shapes:
    h, r ~ N(0, 1); fast and head weights ~ N(0, 0.02) (the weights' init);
    unit final-norm gain; targets uniform over the vocabulary, the last one
    absent."""
    g = torch.Generator(device="cuda").manual_seed(seed)
    rows = n_chunks * b
    h = torch.randn(rows, d, device="cuda", generator=g)
    r = torch.randn(rows, d, device="cuda", generator=g)
    tgt = torch.randint(0, V, (rows,), device="cuda", generator=g, dtype=torch.int32)
    tgt[-1] = -1
    W = [0.02 * torch.randn(f, d, device="cuda", generator=g), 0.02 * torch.randn(f, d, device="cuda", generator=g),
         0.02 * torch.randn(d, f, device="cuda", generator=g)]
    gf = torch.ones(d, device="cuda")
    head = 0.02 * torch.randn(V, d, device="cuda", generator=g)
    return h, r, tgt, W, gf, head


# ops that run only when named with --op (not part of the default list)
OPT_IN = {"meta_grad_top"}


def op_builders(cfg, exp_poly=None):
    """{name: builder}; a builder allocates the op's inputs and returns
    (run, algorithmic flops, algorithmic bytes).  exp_poly: polynomial share
    of the fixed-shift attention forward's exponentials (None = default)."""
    d, f, V, b, k, H, hd = cfg.d_model, cfg.d_ff, cfg.vocab, cfg.b, cfg.k, cfg.n_heads, cfg.head_dim
    S = max(1, 16384 // b) * b
    bf = torch.bfloat16
    dev = "cuda"
    rn = lambda *s, dt=bf: (torch.randn(*s, device=dev) * 0.05).to(dt)
    emp = lambda *s, dt=bf: torch.empty(*s, device=dev, dtype=dt)
    R1 = (S + k + 127) // 128 * 128
    R = (k + b + 127) // 128 * 128
    B = {}

    def gemm(name, M, N, K, a_mn, b_mn, epi, **outs):
        def build():
            A = rn(K, M) if a_mn else rn(M, K)
            Bm = rn(K, N) if b_mn else rn(N, K)
            args = {key: (v() if callable(v) else v) for key, v in outs.items()}
            S, bn = ops.gemm_plan(M, N, K, epi)  # the prefill's tile width and split-K count
            if S > 1:
                ws = torch.empty(S * M * N, device=dev)
                return (lambda: ops.gemm_split(A, Bm, a_mn, b_mn, epi, S, ws, bn=bn, **args)), 2.0 * M * N * K, 0.0
            return (lambda: ops.gemm(A, Bm, a_mn, b_mn, epi, bn=bn, **args)), 2.0 * M * N * K, 0.0
        B[name] = build

    f32 = torch.float32
    gemm("gemm_qkv_bottom", S, 3 * d, d, 0, 0, L.EPI_STORE_BF16, c=lambda: emp(S, 3 * d))
    gemm("gemm_o_bottom", S, d, d, 0, 0, L.EPI_ADD_F32, c=lambda: torch.zeros(S, d, device=dev),
         c2=lambda: torch.zeros(S, d, device=dev))
    gemm("gemm_gateup_bottom", S, 2 * f, d, 0, 0, L.EPI_SWIGLU, c=lambda: emp(S, f))
    gemm("gemm_down_bottom", S, d, f, 0, 0, L.EPI_ADD_F32, c=lambda: torch.zeros(S, d, device=dev))
    gemm("gemm_qkv_top", b, 3 * d, d, 0, 0, L.EPI_STORE_BF16, c=lambda: emp(b, 3 * d))
    gemm("gemm_o_top", b, d, d, 0, 0, L.EPI_ADD_F32, c=lambda: torch.zeros(b, d, device=dev),
         c2=lambda: torch.zeros(b, d, device=dev))
    gemm("gemm_gateup_top", b, 4 * f, d, 0, 0, L.EPI_SWIGLU, c=lambda: emp(b, 2 * f), c2=lambda: emp(b, 4 * f))
    gemm("gemm_down_top", b, d, 2 * f, 0, 0, L.EPI_ADD_F32, c=lambda: torch.zeros(b, d, device=dev))
    gemm("gemm_da_top", b, 2 * f, d, 0, 1, L.EPI_STORE_BF16, c=lambda: emp(b, 2 * f))
    gemm("gemm_dgrad_gateup", b, d, 4 * f, 0, 1, L.EPI_STORE_F32, c=lambda: emp(b, d, dt=f32))
    gemm("gemm_dgrad_o", b, d, d, 0, 1, L.EPI_STORE_BF16, c=lambda: emp(b, d))
    gemm("gemm_dgrad_qkv", b, d, 3 * d, 0, 1, L.EPI_STORE_F32, c=lambda: emp(b, d, dt=f32))
    gemm("gemm_wgrad_gateup_sgd", 2 * f, d, b, 1, 1, L.EPI_SGD, c=lambda: torch.zeros(2 * f, d, device=dev),
         c2=lambda: emp(2 * f, d), c3=lambda: emp(2 * f, d), alpha=1e-2)
    gemm("gemm_wgrad_down_sgd", d, f, b, 1, 1, L.EPI_SGD, c=lambda: torch.zeros(d, f, device=dev),
         c2=lambda: emp(d, f), c3=lambda: emp(d, f), alpha=1e-2)
    gemm("gemm_wgrad_gateup_store", 2 * f, d, b, 1, 1, L.EPI_STORE_F32, c=lambda: torch.zeros(2 * f, d, device=dev))

    def lmhead():
        nt = ops.gemm_ce_tiles(True, b, V)
        A, Bm = rn(b, d), rn(V, d)
        tgt = torch.randint(0, V, (b,), device=dev, dtype=torch.int32)
        pm, ps, zt = emp(nt, b, dt=f32), emp(nt, b, dt=f32), emp(b, dt=f32)
        return (lambda: ops.gemm(A, Bm, 0, 0, L.EPI_CE_FWD, row_i=tgt, part_max=pm, part_sum=ps, target_logit=zt,
                                 part_ld=b)), 2.0 * b * V * d, 0.0
    B["gemm_lmhead_ce_fwd"] = lmhead

    # LM-head backward per vocab chunk (the chunk width the engine picks: dz stays <= 48 MB)
    max_cols = max(256, (48 << 20) // (b * 2) // 256 * 256)
    nvc = -(-V // max_cols)
    Vc = (-(-V // nvc) + 255) // 256 * 256

    def ce_dz():
        A, Bm = rn(b, d), rn(Vc, d)
        lse, scl = torch.zeros(b, device=dev), torch.full((b,), 1.0 / b, device=dev)
        tgt = torch.randint(0, Vc, (b,), device=dev, dtype=torch.int32)
        dz = emp(b, Vc)
        return (lambda: ops.gemm(A, Bm, 0, 0, L.EPI_CE_BWD, c=dz, row_f=lse, row_g=scl, row_i=tgt)), 2.0 * b * Vc * d, 0.0
    B["gemm_ce_dz"] = ce_dz
    gemm("gemm_ce_dh", b, d, Vc, 0, 1, L.EPI_ADD_F32, c=lambda: torch.zeros(b, d, device=dev))

    def swa(name, n, p0, ring, backward=False):
        def build():
            q = rn(n, H * hd)
            kr, vr = rn(ring, H * hd), rn(ring, H * hd)
            o = emp(n, H * hd)
            lse = emp(H, n, dt=f32)
            # the engine passes the bounds of the QK-norm (unit gains: sqrt(head_dim))
            nb = dict(q_norm_max=hd ** 0.5, k_norm_max=hd ** 0.5)
            pairs = band_pairs(p0, n, k)
            if not backward:
                return ((lambda: ops.swa_forward(q, kr, vr, H, hd, p0, k, o, lse, exp_poly=exp_poly, **nb)),
                        4.0 * d * pairs, 0.0)
            ops.swa_forward(q, kr, vr, H, hd, p0, k, o, lse, **nb)
            dout = rn(n, H * hd)
            dq, dk, dv = (torch.empty_like(q) for _ in range(3))
            D = emp(H * n, dt=f32)
            return ((lambda: ops.swa_backward(q, kr, vr, H, hd, p0, k, o, lse, dout, dq, dk, dv, D)),
                    4.0 * d * (pairs + n * (n + 1) // 2), 0.0)
        B[name] = build

    swa("swa_fwd_bottom", S, S, R1)
    swa("swa_fwd_top", b, 8 * b + 64 * 1024 // b * b, R)
    swa("swa_bwd_top", b, 8 * b + 64 * 1024 // b * b, R, backward=True)

    # memory-bound kernels of the prefill
    def rmsnorm():
        x, g1, y, rs = torch.randn(S, d, device=dev), torch.ones(d, device=dev), emp(S, d), emp(S, dt=f32)
        return (lambda: ops.rmsnorm(x, g1, 1e-5, y, rs)), 0.0, S * (4.0 * d + 2.0 * d + 4.0)
    B["rmsnorm_bottom"] = rmsnorm

    def qknorm_rope():
        qkv = rn(S, 3 * d)
        gq, gk = torch.ones(hd, device=dev), torch.ones(hd, device=dev)
        qo, kring, vring = emp(S, d), emp(R1, d), emp(R1, d)
        rq, rk, tab = emp(S, H, dt=f32), emp(S, H, dt=f32), emp(S * hd, dt=f32)
        return ((lambda: ops.qknorm_rope(qkv, S, H, hd, 1e-5, 1e4, gq, gk, qo, kring, vring, rq, rk, tab)), 0.0,
                S * (2.0 * 3 * d * 2 + 8.0 * H + 4.0 * hd))
    B["qknorm_rope_bottom"] = qknorm_rope

    def swiglu_bwd():
        da, gu, dgu = rn(b, 2 * f), rn(b, 4 * f), emp(b, 4 * f)
        return (lambda: ops.swiglu_bwd(da, gu, dgu)), 0.0, b * (2.0 * 2 * f + 2.0 * 4 * f * 2)
    B["swiglu_bwd_top"] = swiglu_bwd

    # generation: one position
    def gemv_gateup():
        w, hv, av, rawv = rn(4 * f, d), rn(d), emp(2 * f), emp(4 * f)
        return (lambda: ops.gemv(2, w, hv, av, raw=rawv)), 0.0, 2.0 * 4 * f * d
    B["gemv_gateup_top"] = gemv_gateup

    def gemv_head():
        w, hv, part, tok = rn(V, d), rn(d), emp(3 * 1184, dt=f32), emp(1, dt=torch.int32)
        return (lambda: ops.gemv(3, w, hv, tok, part=part)), 0.0, 2.0 * V * d
    B["gemv_lmhead_pick"] = gemv_head

    def attn_dec():
        qd, od, lsed = rn(d), emp(d), emp(H, dt=f32)
        wsd = torch.zeros(H * (((k + 127) // 128 + 1) * (hd + 2) + 1), device=dev)
        kdec, vdec = rn(R, d), rn(R, d)
        pdec = 16 * k + 5
        return (lambda: ops.attn_decode(qd, kdec, vdec, H, hd, pdec, k, od, lsed, wsd)), 0.0, 2.0 * 2 * d * k
    B["attn_decode_top"] = attn_dec

    # outer loop: meta-gradient of a fast MLP in the last block over two chunks
    def meta_grad():
        h, r, tgt, W, gf, head = meta_grad_inputs(2, b, d, f, V)
        outs = [torch.empty_like(w) for w in W]
        work = torch.empty(ops.meta_grad_work(2, b, d, f, V), device=dev)
        run = lambda: ops.meta_grad(h, r, tgt, *W, gf, head, 1e-5, 0.5, b, *outs, work=work)
        return run, meta_grad_flops(2, b, d, f, V), 0.0
    B["meta_grad_top"] = meta_grad
    return B


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--config", default="2.7b")
    ap.add_argument("--op", nargs="*", default=None)
    ap.add_argument("--iters", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--exp-poly", type=int, default=None, choices=[0, 2, 4])
    args = ap.parse_args()
    cfg = get_config(args.config)
    builders = op_builders(cfg, args.exp_poly)
    for name in args.op or [n for n in builders if n not in OPT_IN]:
        run, flops, nbytes = builders[name]()
        for _ in range(args.warmup):
            run()
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        for _ in range(args.iters):
            run()
        e1.record()
        ops.sync()
        ms = e0.elapsed_time(e1) / args.iters
        rec = {"op": name, "config": args.config, "ms": ms}
        if name.startswith("swa_fwd"):
            rec.update(exp_poly=args.exp_poly)
        if flops:
            rec.update(tflops=flops / (ms / 1e3) / 1e12, algorithmic_flops=flops)
        if nbytes:
            rec.update(gbps=nbytes / (ms / 1e3) / 1e9, algorithmic_bytes=nbytes)
        print(json.dumps(rec), flush=True)
        del run
        torch.cuda.empty_cache()


if __name__ == "__main__":
    main()
