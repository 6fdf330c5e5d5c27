"""Time single kernels of the prefill loop at a workload's shapes.

    python -m test_long_context_b200.opbench [--config 2.7b] [--op NAME ...] [--iters N]

Each op runs through the op-level C ABI (include/ttt_ops.h) on random
inputs of the exact shapes the engine uses for the named config, timed
with CUDA events after warm-up; one JSON line per op with the average
launch time and the algorithmic TFLOP/s (contractions) or GB/s (the
memory-bound kernels: algorithmic bytes = every operand read and every
result written once).  With --iters 1 --warmup 0 it is
also the small, self-contained command that ncu captures (a few hundred MB
on the device instead of the whole model).
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


def make_ops(cfg):
    d, f, V, b, k, H, hd = cfg.d_model, cfg.d_ff, cfg.vocab, cfg.b, cfg.k, cfg.n_heads, cfg.head_dim
    S = max(1, 16384 // b) * b
    bf = torch.bfloat16
    dev = "cuda"
    rn = lambda *s, dt=bf: (torch.randn(*s, device=dev) * 0.05).to(dt)
    R1 = (S + k + 127) // 128 * 128
    R = (k + b + 127) // 128 * 128
    out = {}

    def gemm(name, M, N, K, a_mn, b_mn, epi, **kw):
        A = rn(K, M) if a_mn else rn(M, K)
        B = rn(K, N) if b_mn else rn(N, K)
        args = dict(kw)

        def run():
            ops.gemm(A, B, a_mn, b_mn, epi, **args)
        out[name] = (run, 2.0 * M * N * K, 0.0)

    gemm("gemm_qkv_bottom", S, 3 * d, d, 0, 0, L.EPI_STORE_BF16, c=torch.empty(S, 3 * d, device=dev, dtype=bf))
    gemm("gemm_gateup_bottom", S, 2 * f, d, 0, 0, L.EPI_SWIGLU, c=torch.empty(S, f, device=dev, dtype=bf))
    gemm("gemm_down_bottom", S, d, f, 0, 0, L.EPI_ADD_F32, c=torch.zeros(S, d, device=dev))
    gemm("gemm_gateup_top", b, 4 * f, d, 0, 0, L.EPI_SWIGLU, c=torch.empty(b, 2 * f, device=dev, dtype=bf),
         c2=torch.empty(b, 4 * f, device=dev, dtype=bf))
    gemm("gemm_down_top", b, d, 2 * f, 0, 0, L.EPI_ADD_F32, c=torch.zeros(b, d, device=dev))
    gemm("gemm_o_top", b, d, d, 0, 0, L.EPI_ADD_F32, c=torch.zeros(b, d, device=dev),
         c2=torch.zeros(b, d, device=dev))
    gemm("gemm_dgrad_gateup", b, d, 4 * f, 0, 1, L.EPI_STORE_F32, c=torch.empty(b, d, device=dev))
    gemm("gemm_wgrad_gateup_sgd", 2 * f, d, b, 1, 1, L.EPI_SGD, c=torch.zeros(2 * f, d, device=dev),
         c2=torch.empty(2 * f, d, device=dev, dtype=bf), c3=torch.empty(2 * f, d, device=dev, dtype=bf), alpha=1e-2)
    gemm("gemm_wgrad_gateup_store", 2 * f, d, b, 1, 1, L.EPI_STORE_F32, c=torch.zeros(2 * f, d, device=dev))
    gemm("gemm_wgrad_gateup_kmajor_store", 2 * f, d, b, 0, 0, L.EPI_STORE_F32, c=torch.zeros(2 * f, d, device=dev))
    nt = ops.gemm_ce_tiles(True, b, V)
    tgt = torch.randint(0, V, (b,), device=dev, dtype=torch.int32)
    gemm("gemm_lmhead_ce_fwd", b, V, d, 0, 0, L.EPI_CE_FWD, row_i=tgt, part_max=torch.empty(nt, b, device=dev),
         part_sum=torch.empty(nt, b, device=dev), target_logit=torch.empty(b, device=dev), part_ld=b)

    def swa(name, n, p0, ring, backward=False):
        q = rn(n, H * hd)
        kr, vr = rn(ring, H * hd), rn(ring, H * hd)
        o = torch.empty(n, H * hd, device=dev, dtype=bf)
        lse = torch.empty(H, n, device=dev)
        ops.swa_forward(q, kr, vr, H, hd, p0, k, o, lse)
        pairs = band_pairs(p0, n, k)
        if not backward:
            out[name] = (lambda: ops.swa_forward(q, kr, vr, H, hd, p0, k, o, lse), 4.0 * d * pairs, 0.0)
        else:
            dout = rn(n, H * hd)
            dq, dk, dv = (torch.empty_like(q) for _ in range(3))
            D = torch.empty(H * n, device=dev)
            out[name] = (lambda: ops.swa_backward(q, kr, vr, H, hd, p0, k, o, lse, dout, dq, dk, dv, D),
                         4.0 * d * (pairs + n * (n + 1) // 2), 0.0)

    gemm("gemm_o_bottom", S, d, d, 0, 0, L.EPI_ADD_F32, c=torch.zeros(S, d, device=dev),
         c2=torch.zeros(S, d, device=dev))
    gemm("gemm_qkv_top", b, 3 * d, d, 0, 0, L.EPI_STORE_BF16, c=torch.empty(b, 3 * d, device=dev, dtype=bf))
    gemm("gemm_da_top", b, 2 * f, d, 0, 1, L.EPI_STORE_BF16, c=torch.empty(b, 2 * f, device=dev, dtype=bf))
    gemm("gemm_dgrad_o", b, d, d, 0, 1, L.EPI_STORE_BF16, c=torch.empty(b, d, device=dev, dtype=bf))
    gemm("gemm_dgrad_qkv", b, d, 3 * d, 0, 1, L.EPI_STORE_F32, c=torch.empty(b, d, device=dev))
    gemm("gemm_wgrad_down_sgd", d, f, b, 1, 1, L.EPI_SGD, c=torch.zeros(d, f, device=dev),
         c2=torch.empty(d, f, device=dev, dtype=bf), c3=torch.empty(d, f, device=dev, dtype=bf), alpha=1e-2)

    # memory-bound kernels (algorithmic bytes)
    x = torch.randn(S, d, device=dev)
    g1 = torch.ones(d, device=dev)
    y = torch.empty(S, d, device=dev, dtype=bf)
    rs = torch.empty(S, device=dev)
    out["rmsnorm_bottom"] = (lambda: ops.rmsnorm(x, g1, 1e-5, y, rs), 0.0, S * (4.0 * d + 2.0 * d + 4.0))
    qkv = rn(S, 3 * d)
    gq, gk = torch.ones(hd, device=dev), torch.ones(hd, device=dev)
    qo = torch.empty(S, d, device=dev, dtype=bf)
    kring, vring = torch.empty(R1, d, device=dev, dtype=bf), torch.empty(R1, d, device=dev, dtype=bf)
    rq, rk = torch.empty(S, H, device=dev), torch.empty(S, H, device=dev)
    tab = torch.empty(S * hd, device=dev)
    out["qknorm_rope_bottom"] = (lambda: ops.qknorm_rope(qkv, S, H, hd, 1e-5, 1e4, gq, gk, qo, kring, vring, rq, rk,
                                                         tab), 0.0, S * (2.0 * 3 * d * 2 + 8.0 * H + 4.0 * hd))
    da = rn(b, 2 * f)
    gu = rn(b, 4 * f)
    dgu = torch.empty(b, 4 * f, device=dev, dtype=bf)
    out["swiglu_bwd_top"] = (lambda: ops.swiglu_bwd(da, gu, dgu), 0.0, b * (2.0 * 2 * f + 2.0 * 4 * f * 2))
    # generation: one position
    wgu = rn(4 * f, d)
    hv = rn(d)
    av = torch.empty(2 * f, device=dev, dtype=bf)
    rawv = torch.empty(4 * f, device=dev, dtype=bf)
    out["gemv_gateup_top"] = (lambda: ops.gemv(2, wgu, hv, av, raw=rawv), 0.0, 2.0 * 4 * f * d)
    whead = rn(V, d)
    part = torch.empty(3 * 1184, device=dev)
    tok = torch.empty(1, device=dev, dtype=torch.int32)
    out["gemv_lmhead_pick"] = (lambda: ops.gemv(3, whead, hv, tok, part=part), 0.0, 2.0 * V * d)
    qd = rn(d)
    od = torch.empty(d, device=dev, dtype=bf)
    lsed = torch.empty(H, device=dev)
    wsd = torch.empty(H * ((k + 127) // 128 + 1) * (hd + 2), device=dev)
    kdec, vdec = rn(R, d), rn(R, d)
    pdec = 16 * k + 5
    out["attn_decode_top"] = (lambda: ops.attn_decode(qd, kdec, vdec, H, hd, pdec, k, od, lsed, wsd), 0.0,
                              2.0 * 2 * d * k)

    swa("swa_fwd_bottom", S, S, R1)
    swa("swa_fwd_top", b, 8 * b + 64 * 1024 // b * b, R)
    swa("swa_bwd_top", b, 8 * b + 64 * 1024 // b * b, R, backward=True)
    return out


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--config", default="2.7b")
    ap.add_argument("--op", nargs="*", default=None)
    ap.add_argument("--iters", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=3)
    args = ap.parse_args()
    cfg = get_config(args.config)
    table = make_ops(cfg)
    names = args.op or list(table)
    for name in names:
        run, flops, nbytes = table[name]
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
        if flops:
            rec.update(tflops=flops / (ms / 1e3) / 1e12, algorithmic_flops=flops)
        if nbytes:
            rec.update(gbps=nbytes / (ms / 1e3) / 1e9, algorithmic_bytes=nbytes)
        print(json.dumps(rec), flush=True)


if __name__ == "__main__":
    main()
