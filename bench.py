#!/usr/bin/env python
"""Prefill throughput of the TTT-E2E loop on B200 (one JSON line on rank 0).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--config 2.7b] [--tokens T] [--no-cpu-baseline]

A step is one full ttt_reset + ttt_prefill over one synthetic sequence of the
workload (every row of the hot path: bottom blocks, chunked forward, loss,
backward through the updated blocks, SGD on the fast MLPs).  Inputs are
seeded synthetic tokens and N(0, 0.02) weights (synth/); the weights (7+ GB
at 2.7B) are far larger than L2, so no flush is needed between steps.

With N > 1 (torchrun) every rank runs an independent replica on its own
sequence (the path does not shard: replicas only); value = tokens of all
ranks / max over ranks of the device time.

--impl reference times the CPU oracle (oracle/) on this machine's host cores on
a bounded sample of the same workload per step: the first CPU_SAMPLE tokens
of the sequence as one chunk (the chunk length set to CPU_SAMPLE), so the
sample runs the whole loop once: forward, loss, backward through the updated
blocks and the SGD step.  The same sample gives cpu_baseline.

After the headline workload, the other workloads (tiny fp32, 125M, 760M) get
one short timing each under "per_config": tokens/s, per-1K-token latency and
the achieved fraction of the roofline.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "prefill tokens/s (2.7B, SWA k=8K, TTT b=1K, T=128K) and % of bf16 tensor peak"
# Tokens of the CPU oracle's bounded sample, run as one chunk of that length
# (forward, loss, backward, update): about ten seconds of fp64 work at 2.7B
# on a 16-core host, most of it widening the weights to fp64.
CPU_SAMPLE = 128
# Workloads timed after the headline one (name -> timed steps)
PER_CONFIG = ("tiny", "125m", "760m")
KC_NAMES = ("gemm", "attn_fwd", "attn_bwd", "other", "norm", "rope", "decode")
# Greedy generation after the headline prefill (the 2.7B decode workload):
# tokens generated, one SGD step on the fast MLPs after every chunk of them
DECODE_TOKENS = 8192


def parse_args():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=3)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--config", default="2.7b")
    ap.add_argument("--tokens", type=int, default=0, help="override T (testing only; not a bench line)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-per-config", action="store_true")
    ap.add_argument("--decode-tokens", type=int, default=DECODE_TOKENS, help="0 skips the decode measurement")
    ap.add_argument("--no-full-attention", action="store_true")
    ap.add_argument("--no-multi-sequence", action="store_true")
    ap.add_argument("--no-meta-grad", action="store_true")
    return ap.parse_args()


def algorithmic_flops(cfg, T):
    """Algorithmic flops of one prefill (2 flops per MAC; attention over the
    eq. (1) band only; backward only for what the method needs; no flash
    recompute):  forward L*(8d^2 + 6df) + n_u*6df + 2dV per token plus
    4d * sum_p min(p+1, k) per block; backward per full chunk: 2dV +
    (n_u-1)(8d^2 + 6df + 12df) + 8df per token (the lowest updated block needs
    only its fast MLP), plus attention 4d*(band + b(b+1)/2) in n_u-1 blocks."""
    L, d, f, V, nu, k, b = cfg.n_layers, cfg.d_model, cfg.d_ff, cfg.vocab, cfg.n_updated, cfg.k, cfg.b
    band = sum(min(p + 1, k) for p in range(T)) if T < 4 * k else (k * (k + 1) // 2 + (T - k) * k)
    fwd = T * (L * (8 * d * d + 6 * d * f) + nu * 6 * d * f + 2 * d * V) + 4 * d * band * L
    full = T // b if T % b == 0 else T // b
    tb = full * b
    bwd = tb * (2 * d * V + (nu - 1) * (8 * d * d + 6 * d * f + 12 * d * f) + 8 * d * f)
    band_full = sum(min(p + 1, k) for p in range(tb)) if tb < 4 * k else (k * (k + 1) // 2 + (tb - k) * k)
    bwd += (nu - 1) * 4 * d * (band_full + full * b * (b + 1) // 2)
    return float(fwd + bwd)


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as fh:
            p = json.load(fh)
        return p, "measured"
    except OSError:
        return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0,
                "sm_max_mhz": 1965.0}, "fallback"


def kernel_source_hash(kc):
    files = {"gemm": ["gemm_tc.cu", "ptx.cuh"], "attn_fwd": ["attention_tc.cu", "ptx.cuh"],
             "attn_bwd": ["attention_tc.cu", "attention.cu", "ptx.cuh"], "other": ["elementwise.cu"],
             "norm": ["elementwise.cu"], "rope": ["elementwise.cu"]}[kc]
    h = hashlib.sha256()
    for f in files:
        with open(os.path.join(ROOT, "test_long_context_b200", "csrc", f), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()[:16]


def traffic_for(kc, workload):
    """DRAM bytes per launch of the kernel class from the committed ncu
    summary, if it was taken on the current source of that kernel."""
    path = os.path.join(ROOT, "profiles", "traffic.json")
    try:
        with open(path) as fh:
            t = json.load(fh)
    except OSError:
        return None
    e = t.get(workload, {}).get(kc)
    if not e or e.get("source_hash") != kernel_source_hash(kc):
        return None
    return e.get("dram_bytes_per_launch")


def rank_tokens(cfg, T, rank):
    """Replica `rank`'s synthetic sequence: an independent problem with its own seed."""
    import synth
    return synth.tokens(cfg, T, seed=cfg.seed + 7919 * rank)


def max_over_ranks(x, dist, world, device):
    """Largest value of x over the ranks (the job's time is its slowest rank's)."""
    if world <= 1:
        return float(x)
    import torch
    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def aggregate_tokens_per_s(world, steps, T, ms):
    """Whole-job throughput: every rank prefills `steps` sequences of T tokens."""
    return world * steps * T / (ms / 1000.0)


class ClockSampler:
    """nvidia-smi sampling of SM clocks and throttle reasons while running."""

    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,clocks_event_reasons.hw_slowdown,"
              "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
              "clocks_event_reasons.sw_power_cap")

    def __init__(self, uuid):
        self.uuid = uuid
        self.proc = None
        self.path = os.path.join("/tmp", f"ttt_clocks_{os.getpid()}.csv")

    def start(self):
        try:
            self.fh = open(self.path, "w")
            self.proc = subprocess.Popen(["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                                          "-lms", "200", "-i", self.uuid], stdout=self.fh, stderr=subprocess.DEVNULL)
        except OSError:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return None
        time.sleep(0.3)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        self.fh.close()
        sm, mx, reasons = [], 0.0, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        with open(self.path) as fh:
            for line in fh:
                parts = [p.strip() for p in line.split(",")]
                if len(parts) < 8:
                    continue
                try:
                    sm.append(float(parts[0]))
                    mx = max(mx, float(parts[1]))
                except ValueError:
                    continue
                for name, v in zip(names, parts[4:8]):
                    if v.lower().startswith("active"):
                        reasons.add(name)
        os.unlink(self.path)
        if not sm:
            return None
        loaded = [s for s in sm if s > 0.5 * max(sm)] or sm
        return {"sm_mhz": statistics.median(loaded), "sm_max_mhz": mx, "reasons": sorted(reasons),
                "samples": len(sm)}


def latency_by_tokens(ctx, tok_dev, losses, T, stream, lengths=(8192, 16384, 32768, 65536)):
    """Per-1K-token prefill latency (ms) of one prefill of each shorter prefix
    of the same sequence and of the whole sequence, all without per-launch
    timing events: the cost per token should stay flat once the window is
    full."""
    import torch
    out = {}
    for n in [m for m in lengths if m < T] + [T]:
        ctx.reset()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        ctx.prefill(tok_dev[:n], losses[:n], sync=False)
        e1.record(stream)
        ctx.sync()
        out[str(n)] = e0.elapsed_time(e1) / (n / 1000.0)
    return out


def marginal_latency(by_T):
    """Per-1K-token cost of the tokens added between consecutive prefix
    lengths, (t(T2) - t(T1)) / (T2 - T1): flat once the window is full
    (reading notes, eq. (11)), while the average over a whole prefix still
    carries the cheaper first k positions."""
    pts = sorted((int(n), v * int(n) / 1000.0) for n, v in by_T.items())
    return {f"{a}-{b}": (tb - ta) / ((b - a) / 1000.0) for (a, ta), (b, tb) in zip(pts, pts[1:])}


def workload_name(cfg, T):
    return (f"{cfg.name} TTT-E2E prefill: L={cfg.n_layers} d={cfg.d_model} H={cfg.n_heads}x{cfg.head_dim} "
            f"f={cfg.d_ff} V={cfg.vocab} n_u={cfg.n_updated} T={T} k={cfg.k} b={cfg.b} batch=1")


def config_dict(cfg, T, n):
    return {"workload": workload_name(cfg, T), "tokens_per_sequence": T, "window": cfg.k, "chunk": cfg.b,
            "updated_blocks": cfg.n_updated, "sequences_per_gpu": 1, "parallelism": f"replicas{n}",
            "l2": "inputs larger than L2 (7 GB of bf16 weights streamed per step), no flush"}


def cpu_baseline(cfg, weights_arrays, toks, sample_tokens):
    """The oracle as it stands on this host's cores: the first `sample_tokens`
    tokens as one chunk of that length, so the sample runs forward, loss,
    backward and the SGD update once."""
    import numpy as np

    import oracle
    m = oracle.Model(cfg, weights_arrays)
    t0 = time.perf_counter()
    oracle.prefill(m, np.asarray(toks[:sample_tokens]), b=sample_tokens)
    dt = time.perf_counter() - t0
    cores = os.cpu_count()
    return {"value": sample_tokens / dt, "unit": "tokens/s", "cores": cores, "kind": "oracle",
            "sample": (f"oracle (fp64 numpy, BLAS threads = {cores}): the first {sample_tokens} tokens of the same "
                       f"sequence as one chunk of {sample_tokens} (the workload's chunk is {cfg.b}): forward, loss, "
                       f"backward through the {cfg.n_updated} updated blocks and the SGD step, including the "
                       f"per-call widening of the weights to fp64; the window is not yet full"),
            "seconds": dt}


def cpu_baseline_sample_text(cfg, sample):
    return (f"first {sample} tokens as one chunk of {sample} (forward, loss, backward, SGD update)")


def run_reference(args, cfg, T):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    import synth
    w = synth.make_weights(cfg, keep_bits=False)
    toks = synth.tokens(cfg, T)
    sample = min(CPU_SAMPLE, T)
    for _ in range(args.warmup):
        cpu_baseline(cfg, w.arrays, toks, sample)
    times = []
    for _ in range(args.steps):
        times.append(cpu_baseline(cfg, w.arrays, toks, sample)["seconds"])
    tot = sum(times)
    value = args.steps * sample / tot
    cores = os.cpu_count()
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1000 * tot / args.steps,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic (seeded Zipf + repeated spans; N(0,0.02) weights)", "config": config_dict(cfg, T, 1),
            "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": cores, "kind": "oracle",
                             "sample": cpu_baseline_sample_text(cfg, sample) + " per step"},
            "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


def time_decode(ctx, cfg, tok_dev, T, n_tokens, stream):
    """Greedy generation of n_tokens after a prefill of the T-token prompt
    (the 2.7B decode workload): one ttt_decode call per chunk of b tokens,
    each bracketed by CUDA events on the context's stream.  Reports tokens/s,
    per-token latency, the time the chunk updates add (from the per-class
    timing: the backward and SGD kernels run only at chunk ends), and the
    HBM roofline of the per-position kernels (their algorithmic bytes: every
    weight read once per position plus the window's keys and values)."""
    import torch
    peaks, src = load_peaks()
    b = cfg.b
    ctx.reset()
    ctx.prefill(tok_dev, sync=False)
    ctx.decode(64, sync=True)  # warm-up (kernels loaded, first pick taken)
    ctx.reset()
    ctx.prefill(tok_dev, sync=False)
    ctx.sync()
    toks = torch.empty(n_tokens, device="cuda", dtype=torch.int32)
    evs = [torch.cuda.Event(enable_timing=True) for _ in range(n_tokens // b + 2)]
    evs[0].record(stream)
    done, i = 0, 0
    while done < n_tokens:
        n = min(b - (T + done) % b, n_tokens - done)  # up to the next chunk end
        ctx.decode(n, tokens=toks[done:done + n], sync=False)
        done += n
        i += 1
        evs[i].record(stream)
    ctx.sync()
    total_ms = evs[0].elapsed_time(evs[i])
    per_chunk = [evs[j].elapsed_time(evs[j + 1]) for j in range(i)]
    # one more chunk with per-launch timing: bytes and time of the per-position
    # kernels, and the time of the chunk's update (every other class)
    ctx.timing_enable(True)
    ctx.decode(b, sync=False)
    timing = ctx.timing_read()
    ctx.timing_enable(False)
    dms, dn, dbytes = timing["decode"]
    upd_ms = sum(v[0] for k, v in timing.items() if k != "decode")
    n_upd = (T + n_tokens) // b - T // b
    return {"workload": f"{cfg.name} greedy decode of {n_tokens} tokens after a {T}-token prefill, window {cfg.k}, "
                        f"one SGD step on the fast MLPs after every {b} generated positions",
            "tokens": n_tokens, "tokens_per_s": n_tokens / (total_ms / 1000.0), "ms_per_token": total_ms / n_tokens,
            "updates": n_upd, "update_ms_each": upd_ms,
            "ms_per_chunk_of_tokens": per_chunk,
            "launches_per_token": dn / b,
            "roofline": {"bound": "hbm", "kernel": "decode (per-position kernels)",
                         "achieved": dbytes / (dms / 1000.0) / 1e9, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                         "frac": dbytes / (dms / 1000.0) / 1e9 / peaks["hbm_gbs"],
                         "algorithmic_bytes_per_token": dbytes / b, "peak_source": src,
                         "note": "per-launch events of one further chunk of b tokens"},
            "first_tokens": toks[:8].cpu().tolist()}


def time_full_attention(cfg, gw, tok_dev, T, stream, ttt_ms):
    """The same model as a plain full-attention Transformer prefill: window
    k = T (every query sees all earlier positions) and eta = 0, so no chunk
    is updated and the engine runs no backward.  One prefill of the whole
    sequence after a short warm-up, timed with CUDA events; the ratio to the
    TTT prefill's time is the comparison the pages make at 128K (reading
    notes §11.1)."""
    import torch

    from test_long_context_b200.context import Context
    ctx = Context(cfg, gw, k=T, eta=0.0, stream=stream)
    losses = torch.empty(T, device="cuda")
    ctx.prefill(tok_dev[:4096], losses[:4096], sync=True)  # warm-up
    ctx.reset()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    ctx.prefill(tok_dev, losses, sync=False)
    e1.record(stream)
    ctx.sync()
    ms = e0.elapsed_time(e1)
    ok = bool(torch.isfinite(losses[:-1]).all().item())
    ctx.close()
    torch.cuda.empty_cache()
    return {"workload": f"{cfg.name} full-attention prefill (window k = T = {T}, eta = 0: no update, no backward), "
                        "same model and tokens", "tokens_per_s": T / (ms / 1000.0), "ms": ms,
            "ms_per_1k_tokens": ms / (T / 1000.0), "ttt_prefill_speedup": ms / ttt_ms, "finite_losses": ok}


def time_multi_sequence(cfg, gw, n_seq, T_seq, ttt_tokens_per_s):
    """The batch the pages measure with: 128K tokens per batch as n_seq
    independent sequences of T_seq tokens (4 x 32K), each with its own fast
    weights, attention state and context, prefilled at the same time on its
    own CUDA stream (static weights shared).  Time from an event before the
    first launch to the last stream's end; throughput = all tokens / that."""
    import torch

    import synth
    from test_long_context_b200.context import Context
    streams = [torch.cuda.Stream() for _ in range(n_seq)]
    ctxs = [Context(cfg, gw, stream=st) for st in streams]
    toks = [torch.from_numpy(synth.tokens(cfg, T_seq, seed=cfg.seed + 101 * (i + 1))).cuda() for i in range(n_seq)]
    losses = [torch.empty(T_seq, device="cuda") for _ in range(n_seq)]

    def run():
        start = torch.cuda.Event(enable_timing=True)
        start.record(torch.cuda.current_stream())
        ends = []
        for c, t, l, st in zip(ctxs, toks, losses, streams):
            st.wait_event(start)
            c.reset()
            c.prefill(t, l, sync=False)
            e = torch.cuda.Event(enable_timing=True)
            e.record(st)
            ends.append(e)
        for c in ctxs:
            c.sync()
        return max(start.elapsed_time(e) for e in ends)

    run()  # warm-up
    ms = run()
    ok = all(bool(torch.isfinite(l[:-1]).all().item()) for l in losses)
    for c in ctxs:
        c.close()
    torch.cuda.empty_cache()
    tps = n_seq * T_seq / (ms / 1000.0)
    return {"workload": f"{cfg.name} prefill of {n_seq} independent sequences x {T_seq} tokens (window {cfg.k}, chunk "
                        f"{cfg.b}), one context and CUDA stream per sequence, prefilled concurrently",
            "tokens_per_s": tps, "ms": ms, "ms_per_1k_tokens": ms / (n_seq * T_seq / 1000.0),
            "vs_one_sequence_of_the_same_tokens": tps / ttt_tokens_per_s, "finite_losses": ok}


def time_meta_grad(cfg, n_chunks=2, steps=2, warmup=1):
    """The outer loop's meta-gradient (eq. (7) of the reading notes, §4) for a
    fast MLP in the last block at the model's shapes: n_chunks chunks of b
    rows through ttt_op_meta_grad (fp32), inputs seeded and resident, timed
    with CUDA events; achieved = its GEMM flops / time against the fp32 FMA
    peak of the SIMT kernels."""
    import torch

    from test_long_context_b200 import ops
    from test_long_context_b200.opbench import meta_grad_flops, meta_grad_inputs
    b, d, f, V = cfg.b, cfg.d_model, cfg.d_ff, cfg.vocab
    h, r, tgt, W, gf, head = meta_grad_inputs(n_chunks, b, d, f, V)
    outs = [torch.empty_like(w) for w in W]
    losses = torch.empty(n_chunks * b, device="cuda")
    work = torch.empty(ops.meta_grad_work(n_chunks, b, d, f, V), device="cuda")
    run = lambda: ops.meta_grad(h, r, tgt, *W, gf, head, cfg.norm_eps, cfg.eta, b, *outs, losses=losses, work=work)
    for _ in range(warmup):
        run()
    ops.sync()
    stream = torch.cuda.current_stream()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(steps):
        run()
    e1.record(stream)
    ops.sync()
    ms = e0.elapsed_time(e1) / steps
    ok = all(bool(torch.isfinite(o).all().item()) for o in outs)
    flops = meta_grad_flops(n_chunks, b, d, f, V)
    peaks, src = load_peaks()
    peak = 148 * 128 * 2 * peaks.get("sm_max_mhz", 1965.0) * 1e6 / 1e12
    del h, r, W, head, work, outs
    torch.cuda.empty_cache()
    return {"workload": f"{cfg.name} fast-MLP meta-gradient, eq. (7): {n_chunks} chunks x {b} rows, d={d} f={f} "
                        f"V={V}, eta={cfg.eta}, fp32", "ms": ms, "steps": steps, "warmup": warmup,
            "algorithmic_tflop": flops / 1e12,
            "roofline": {"bound": "alu", "achieved": flops / (ms / 1000.0) / 1e12, "peak": peak, "unit": "TFLOP/s",
                         "frac": flops / (ms / 1000.0) / 1e12 / peak, "peak_source": src},
            "finite": ok}


def time_config(name, steps=3, warmup=2):
    """Short timing of one more workload (its own T, k, b, dtype) on this GPU:
    tokens/s, per-1K-token latency and the achieved fraction of its roofline
    (bf16: algorithmic flops against the sustained bf16 peak; fp32: against
    the fp32 FMA peak of the SIMT kernels)."""
    import torch

    import synth
    from test_long_context_b200.context import Context, upload_weights
    cfg = synth.get_config(name)
    T = cfg.T
    gw = {}
    for n, arr, bits in synth.iter_weights(cfg):
        gw.update(upload_weights([(n, arr, bits)], cfg.dtype))
    tok = torch.from_numpy(synth.tokens(cfg)).cuda()
    stream = torch.cuda.current_stream()
    ctx = Context(cfg, gw, stream=stream)
    losses = torch.empty(T, device="cuda")
    for _ in range(warmup):
        ctx.reset()
        ctx.prefill(tok, losses, sync=False)
    ctx.sync()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(steps):
        ctx.reset()
        ctx.prefill(tok, losses, sync=False)
    e1.record(stream)
    ctx.sync()
    ms = e0.elapsed_time(e1) / steps
    ok = bool(torch.isfinite(losses[:-1]).all().item())
    ctx.close()
    del gw
    torch.cuda.empty_cache()
    peaks, src = load_peaks()
    flops = algorithmic_flops(cfg, T)
    if cfg.dtype == "f32":
        peak = 148 * 128 * 2 * peaks.get("sm_max_mhz", 1965.0) * 1e6 / 1e12
        bound = "alu"
    else:
        peak, bound = peaks["bf16_tflops_sustained"], "tensor"
    achieved = flops / (ms / 1000.0) / 1e12
    return {"workload": workload_name(cfg, T), "dtype": cfg.dtype, "tokens_per_s": T / (ms / 1000.0),
            "ms_per_step": ms, "ms_per_1k_tokens": ms / (T / 1000.0), "steps": steps, "warmup": warmup,
            "algorithmic_tflop_per_step": flops / 1e12,
            "roofline": {"bound": bound, "achieved": achieved, "peak": peak, "unit": "TFLOP/s",
                         "frac": achieved / peak, "peak_source": src},
            "finite_losses": ok}


def main():
    args = parse_args()
    if os.environ.get("TTT_BENCH_WATCHDOG"):
        import faulthandler
        faulthandler.dump_traceback_later(int(os.environ["TTT_BENCH_WATCHDOG"]), repeat=True, file=sys.stderr)
    import synth
    cfg = synth.get_config(args.config)
    T = args.tokens or cfg.T
    if args.impl == "reference":
        return run_reference(args, cfg, T)

    import numpy as np
    import torch
    import torch.distributed as dist

    from test_long_context_b200.context import Context, upload_weights

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world != args.gpus:
        raise SystemExit(f"--gpus {args.gpus} but WORLD_SIZE={world}")
    torch.cuda.set_device(local)
    if world > 1:
        from datetime import timedelta
        dist.init_process_group("nccl", timeout=timedelta(seconds=600), device_id=torch.device("cuda", local))

    want_cpu = rank == 0 and world == 1 and not args.no_cpu_baseline
    keep = {}
    gw = {}
    for name, arr, bits in synth.iter_weights(cfg):
        gw.update(upload_weights([(name, arr, bits)], cfg.dtype))
        if want_cpu:
            keep[name] = arr
    toks = rank_tokens(cfg, T, rank)
    tok_dev = torch.from_numpy(toks).cuda()
    stream = torch.cuda.current_stream()
    ctx = Context(cfg, gw, stream=stream)
    losses = torch.empty(T, device="cuda")

    def step():
        ctx.reset()
        ctx.prefill(tok_dev, losses, sync=False)

    for _ in range(args.warmup):
        step()
    ctx.sync()
    if not torch.isfinite(losses[:-1]).all():
        raise SystemExit("non-finite losses")

    uuid = str(torch.cuda.get_device_properties(local).uuid)
    uuid = uuid if uuid.startswith("GPU-") else "GPU-" + uuid
    clocks = ClockSampler(uuid)
    ctx.timing_enable(True)
    n0 = ctx.launch_count()
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    clocks.start()
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    ev0.record(stream)
    for _ in range(args.steps):
        step()
    ev1.record(stream)
    ctx.sync()
    torch.cuda.synchronize()
    clk = clocks.stop()
    if world > 1:
        dist.barrier()
    ms = ev0.elapsed_time(ev1)
    launches = ctx.launch_count() - n0
    timing = ctx.timing_read()
    ctx.timing_enable(False)
    ms = max_over_ranks(ms, dist, world, "cuda")

    # end to end through the public API: pinned host tokens in, losses out
    e2e = None
    if not args.no_e2e:
        tok_host = torch.from_numpy(toks).pin_memory()
        loss_host = torch.empty(T, dtype=torch.float32).pin_memory()
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(args.steps):
            tok_dev.copy_(tok_host, non_blocking=True)
            ctx.reset()
            ctx.prefill(tok_dev, losses, sync=False)
            loss_host.copy_(losses, non_blocking=True)
        e1.record(stream)
        ctx.sync()
        torch.cuda.synchronize()
        ems = max_over_ranks(e0.elapsed_time(e1), dist, world, "cuda")
        e2e = {"value": aggregate_tokens_per_s(world, args.steps, T, ems), "unit": "tokens/s",
               "h2d_bytes_per_step": int(tok_host.numel() * 4), "d2h_bytes_per_step": int(loss_host.numel() * 4),
               "ms_per_step": ems / args.steps}

    by_T = latency_by_tokens(ctx, tok_dev, losses, T, stream)
    dec = None
    if args.decode_tokens > 0 and not args.tokens and args.config == "2.7b":
        dec = time_decode(ctx, cfg, tok_dev, T, args.decode_tokens, stream)

    if rank == 0:
        peaks, peak_src = load_peaks()
        value = aggregate_tokens_per_s(world, args.steps, T, ms)
        flops_step = algorithmic_flops(cfg, T)
        tensor_peak = peaks["bf16_tflops_sustained"]
        classes = {}
        for name in KC_NAMES:
            tms, tn, tfl = timing[name]
            classes[name] = {"ms_per_step": tms / args.steps, "launches_per_step": tn / args.steps,
                             "share": tms / max(1e-9, sum(v[0] for v in timing.values())),
                             "tflops": (tfl / (tms / 1000.0) / 1e12) if tms > 0 and tfl > 0 else None}
        dom = max(KC_NAMES[:3], key=lambda n: timing[n][0])
        tms, tn, tfl = timing[dom]
        achieved = tfl / (tms / 1000.0) / 1e12
        if cfg.dtype == "f32":
            # fp32 mode runs SIMT FMA kernels: 148 SMs x 128 FP32 lanes x 2 flop x max SM clock
            peak = 148 * 128 * 2 * peaks.get("sm_max_mhz", 1965.0) * 1e6 / 1e12
            bound, note = "alu", "fp32 FMA peak from unit counts and the max SM clock"
        else:
            peak, bound, note = tensor_peak, "tensor", f"bf16 dense, sustained ({peak_src})"
        per_launch_flops = tfl / max(tn, 1)
        traffic = traffic_for(dom, args.config)
        roof = {"bound": bound, "kernel": dom, "achieved": achieved, "peak": peak, "unit": "TFLOP/s",
                "frac": achieved / peak, "traffic": traffic, "algorithmic_flops_per_launch": per_launch_flops,
                "avg_launch_ms": tms / max(tn, 1), "peak_source": note}
        line = {"metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world, "steps": args.steps,
                "warmup": args.warmup, "ms_per_step": ms / args.steps, "higher_is_better": True, "scaling": "weak",
                "vs_baseline": None, "dtype": cfg.dtype,
                "data": "synthetic (seeded Zipf(1.1) tokens + repeated 64-token spans; N(0,0.02) weights)",
                "config": config_dict(cfg, T, world),
                "ms_per_1k_tokens": (ms / args.steps) / (T / 1000.0),
                "ms_per_1k_tokens_by_T": by_T,
                "ms_per_1k_tokens_marginal": marginal_latency(by_T),
                "tensor_peak_frac": flops_step * world * args.steps / (ms / 1000.0) / 1e12 / tensor_peak,
                "algorithmic_tflop_per_step": flops_step / 1e12,
                "roofline": roof, "kernel_classes": classes, "gpu_launches": int(launches),
                "clocks": clk, "e2e": e2e, "decode": dec}
    ctx.close()
    torch.cuda.empty_cache()
    full = multi = meta = None
    if rank == 0 and not args.no_meta_grad and world == 1 and args.config == "2.7b" and not args.tokens:
        try:
            meta = time_meta_grad(cfg)
        except Exception as e:  # an optional arm must not cost the headline line
            meta = {"unavailable": f"{type(e).__name__}: {e}"}
    if rank == 0 and not args.no_full_attention and world == 1 and args.config == "2.7b" and not args.tokens:
        full = time_full_attention(cfg, gw, tok_dev, T, stream, ms / args.steps)
    if rank == 0 and not args.no_multi_sequence and world == 1 and args.config == "2.7b" and not args.tokens:
        multi = time_multi_sequence(cfg, gw, 4, T // 4, aggregate_tokens_per_s(1, args.steps, T, ms))
    del gw
    torch.cuda.empty_cache()
    if rank == 0:
        line["full_attention"] = full
        line["multi_sequence"] = multi
        line["meta_grad"] = meta
        if not args.no_per_config and world == 1 and args.config == "2.7b" and not args.tokens:
            line["per_config"] = {name: time_config(name) for name in PER_CONFIG}
        if want_cpu:
            line["cpu_baseline"] = cpu_baseline(cfg, keep, toks, min(CPU_SAMPLE, T))
            line["cpu_baseline"].pop("seconds", None)
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
