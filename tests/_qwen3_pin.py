"""Independent library model used to pin the oracle's forward pass.

transformers' Qwen3 decoder has the same block as the pages' backbone
(pre-RMSNorm, per-head QK RMSNorm before rotate-half RoPE, SwiGLU MLP,
untied head) and supports a sliding window with the same edge convention
(key j visible to query p iff p - k < j <= p).  The oracle's dual MLP
(static + fast, outputs summed) equals one SwiGLU MLP whose hidden units are
the concatenation of both; blocks without a fast MLP get zero-padded hidden
units, which contribute exactly zero."""
import numpy as np
import torch


def build(cfg, arrays, fast=None, sliding=True):
    from transformers import Qwen3Config, Qwen3ForCausalLM

    L, d, H, hd, f, V = cfg.n_layers, cfg.d_model, cfg.n_heads, cfg.head_dim, cfg.d_ff, cfg.vocab
    qc = Qwen3Config(vocab_size=V, hidden_size=d, intermediate_size=2 * f, num_hidden_layers=L,
                     num_attention_heads=H, num_key_value_heads=H, head_dim=hd, rms_norm_eps=cfg.norm_eps,
                     rope_parameters={"rope_theta": cfg.rope_theta, "rope_type": "default"},
                     tie_word_embeddings=False, attention_bias=False, use_sliding_window=sliding,
                     sliding_window=cfg.k if sliding else None, max_window_layers=0,
                     layer_types=["sliding_attention" if sliding else "full_attention"] * L,
                     max_position_embeddings=max(4096, cfg.T))
    qc._attn_implementation = "eager"
    m = Qwen3ForCausalLM(qc).double().eval()
    t = lambda a: torch.tensor(np.asarray(a, dtype=np.float64))
    top = range(L - cfg.n_updated, L)
    with torch.no_grad():
        m.model.embed_tokens.weight.copy_(t(arrays["embed"]))
        m.lm_head.weight.copy_(t(arrays["lm_head"]))
        m.model.norm.weight.copy_(t(arrays["final_norm"]))
        for l, blk in enumerate(m.model.layers):
            p = f"layers.{l}."
            blk.input_layernorm.weight.copy_(t(arrays[p + "attn_norm"]))
            blk.post_attention_layernorm.weight.copy_(t(arrays[p + "mlp_norm"]))
            a = blk.self_attn
            a.q_proj.weight.copy_(t(arrays[p + "wq"]))
            a.k_proj.weight.copy_(t(arrays[p + "wk"]))
            a.v_proj.weight.copy_(t(arrays[p + "wv"]))
            a.o_proj.weight.copy_(t(arrays[p + "wo"]))
            a.q_norm.weight.copy_(t(arrays[p + "q_norm"]))
            a.k_norm.weight.copy_(t(arrays[p + "k_norm"]))
            if l in top:
                src = fast[l] if fast is not None else {n: arrays[f"fast.{l}.{n}"] for n in ("w_gate", "w_up", "w_down")}
                fg, fu, fd = src["w_gate"], src["w_up"], src["w_down"]
            else:
                fg = fu = np.zeros((f, d))
                fd = np.zeros((d, f))
            blk.mlp.gate_proj.weight.copy_(t(np.concatenate([arrays[p + "w_gate"], fg], 0)))
            blk.mlp.up_proj.weight.copy_(t(np.concatenate([arrays[p + "w_up"], fu], 0)))
            blk.mlp.down_proj.weight.copy_(t(np.concatenate([arrays[p + "w_down"], fd], 1)))
    return m


def losses(m, toks):
    """Per-position next-token CE (natural log); last position NaN."""
    ids = torch.tensor(np.asarray(toks, dtype=np.int64))[None]
    with torch.no_grad():
        z = m(input_ids=ids).logits[0]
    lp = torch.log_softmax(z, -1)
    out = np.full(len(toks), np.nan)
    out[:-1] = (-lp[:-1].gather(1, ids[0, 1:, None])[:, 0]).numpy()
    return out
