"""The bf16 noise floor of the prefill forward — TEST INFRASTRUCTURE ONLY.

Only ``tests/`` (and the scripts under ``tests/golden/`` that write stored
values) may import this module.  It shares no code with the CUDA library.

The bf16 workloads keep activations in bf16 where they feed a tensor-core
product (the benchmark spec's bf16 mode: bf16 operands, fp32 accumulation, fp32
norms, softmax and residual).  Even an exact implementation of that mode
differs from the fp64 oracle by the rounding of those stored tensors.  This
module runs the oracle's own forward (its functions, in the same order as
``ttt_oracle.forward_chunk``) in fp64 twice on the same inputs: once exactly,
once with every tensor that the bf16 pipeline stores as bf16 rounded to bf16
(round to nearest, ties to even) at that point.  The difference of the
per-token losses is the floor below which no bf16 pipeline with these
rounding points can go; it is a property of the storage format, not of any
kernel.

Rounding points (``SITES``), in forward order per block:
  h    the attention RMSNorm output (A operand of the q/k/v projection)
  qkv  q, k, v as the projection stores them
  qk   q and k after QK-norm and RoPE (operands of S = q k^T; k is cached)
  P    the unnormalised attention probabilities (operand of P V)
  o    the attention output (A operand of the output projection)
  h2   the MLP RMSNorm output (A operand of the gate/up projections)
  a    the SwiGLU activations (A operand of the down projection)
and once at the end:
  hf   the final RMSNorm output (A operand of the LM head)
"""
from __future__ import annotations

import numpy as np

from . import ttt_oracle as O

SITES = ("h", "qkv", "qk", "P", "o", "h2", "a", "hf")


def bf16_round(x):
    """fp64 -> fp32 -> bf16 (round to nearest, ties to even) -> fp64.
    NaN and infinities are not expected here."""
    a32 = np.ascontiguousarray(x, dtype=np.float32)
    u = a32.view(np.uint32).astype(np.uint64)
    r = ((u + 0x7FFF + ((u >> 16) & 1)) >> 16) << 16
    return r.astype(np.uint32).view(np.float32).astype(np.float64).reshape(np.shape(x))


def forward_losses(model, W, toks, n, sites=SITES):
    """Per-token losses of positions 0 .. n-1 (tokens[1 .. n] as targets) in
    one forward pass from position 0 with fast weights W, rounding to bf16
    at ``sites``.  With ``sites=()`` this is the oracle's forward."""
    cfg = model.cfg
    R = (lambda s, x: bf16_round(x) if s in sites else x)
    L, d, H, hd, eps = cfg.n_layers, cfg.d_model, cfg.n_heads, cfg.head_dim, cfg.norm_eps
    pos = np.arange(n)
    cos, sin = O.rope_tables(pos, hd, cfg.rope_theta)
    mask = O.window_mask(pos, pos, cfg.k)
    toks = np.asarray(toks, dtype=np.int64)
    x = model.rows("embed", toks[:n])
    for l in range(L):
        pre = f"layers.{l}."
        h = R("h", O.rmsnorm(x, model[pre + "attn_norm"], eps)[0])
        q = R("qkv", h @ model[pre + "wq"].T).reshape(n, H, hd)
        k = R("qkv", h @ model[pre + "wk"].T).reshape(n, H, hd)
        v = R("qkv", h @ model[pre + "wv"].T).reshape(n, H, hd)
        qr = R("qk", O.rope(O.rmsnorm(q, model[pre + "q_norm"], eps)[0], cos, sin))
        kr = R("qk", O.rope(O.rmsnorm(k, model[pre + "k_norm"], eps)[0], cos, sin))
        s = np.einsum("qhd,khd->hqk", qr, kr) / np.sqrt(hd)
        s = np.where(mask[None], s, -np.inf)
        p = np.exp(s - s.max(-1, keepdims=True))
        o = np.einsum("hqk,khd->qhd", R("P", p), v) / p.sum(-1, keepdims=True).transpose(1, 0, 2)
        x = x + R("o", o).reshape(n, d) @ model[pre + "wo"].T
        h2 = R("h2", O.rmsnorm(x, model[pre + "mlp_norm"], eps)[0])

        def mlp(wg, wu, wd):
            g, u = h2 @ wg.T, h2 @ wu.T
            return R("a", g * O.sigmoid(g) * u) @ wd.T

        y = mlp(model[pre + "w_gate"], model[pre + "w_up"], model[pre + "w_down"])
        if l in W:
            y = y + mlp(W[l]["w_gate"], W[l]["w_up"], W[l]["w_down"])
        x = x + y
    hf = R("hf", O.rmsnorm(x, model["final_norm"], eps)[0])
    return O.log_softmax_ce(hf @ model["lm_head"].T, toks[1:n + 1])[0]


def floor(model, toks, n, sites=SITES):
    """|rounded - exact| per-token loss of positions 0 .. n-1 with W_init
    (the first chunk when n <= b: scored before any update)."""
    W = O.init_fast(model)
    exact = forward_losses(model, W, toks, n, ())
    rounded = forward_losses(model, W, toks, n, sites)
    return np.abs(rounded - exact)
