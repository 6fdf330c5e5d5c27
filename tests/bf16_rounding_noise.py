"""How much per-token loss error does bf16 rounding of the activations alone
cause?  The fp64 CPU model of the forward pass (the oracle's functions) is
run twice on the same inputs: exactly, and with the tensors that the bf16
GPU path stores in bf16 rounded to bf16 (round to nearest even) at the same
points: the attention-norm output, the q/k/v projections, q and k after
QK-norm and RoPE, the unnormalised attention probabilities, the attention
output, the MLP-norm output, the SwiGLU activations and the final-norm
output.  Weights are the same bf16-exact values in both runs.  The
difference of the per-token losses is the noise floor of any bf16 pipeline
with these rounding points; the test tolerances of the full-size parity
tests are read against it.

    python -m tests.bf16_rounding_noise [config] [tokens]

Test infrastructure: reads the oracle, never the CUDA library.
"""
import sys

import numpy as np

import synth
from oracle import ttt_oracle as O


def bf16_round(x):
    a32 = np.asarray(x, dtype=np.float32)
    u = a32.view(np.uint32).astype(np.uint64)
    r = ((u + 0x7FFF + ((u >> 16) & 1)) >> 16) << 16
    return r.astype(np.uint32).view(np.float32).astype(np.float64)


SITES = ("h", "qkv", "qk", "P", "o", "h2", "a", "hf")


def forward_losses(cfg, model, W, toks, n, sites):
    """Per-token losses of positions 0 .. n-1 (one forward pass from the start,
    fast weights W) with bf16 rounding at `sites`."""
    R = (lambda s, x: bf16_round(x) if s in sites else x)
    L, d, H, hd, eps = cfg.n_layers, cfg.d_model, cfg.n_heads, cfg.head_dim, cfg.norm_eps
    pos = np.arange(n)
    cos, sin = O.rope_tables(pos, hd, cfg.rope_theta)
    mask = O.window_mask(pos, pos, cfg.k)
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


def main():
    name = sys.argv[1] if len(sys.argv) > 1 else "125m"
    n = int(sys.argv[2]) if len(sys.argv) > 2 else 512
    cfg = synth.get_config(name)
    w = synth.make_weights(cfg)
    toks = synth.tokens(cfg)[:n + 1]
    model = O.Model(cfg, w.arrays)
    W = O.init_fast(model)
    exact = forward_losses(cfg, model, W, toks, n, ())
    rounded = forward_losses(cfg, model, W, toks, n, SITES)
    d = np.abs(rounded - exact)
    print(f"{name}, {n} tokens: per-token |loss error| max {d.max():.4f}, p99.5 {np.percentile(d, 99.5):.4f}, "
          f"mean {d.mean():.4f}")


if __name__ == "__main__":
    main()
