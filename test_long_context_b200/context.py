"""torch-facing wrapper of the C ABI in include/ttt.h (argument marshalling
only).  Weights are torch CUDA tensors that must stay alive while the
context exists; the wrapper keeps references to them."""
from __future__ import annotations

import ctypes

import numpy as np
import torch

from . import _lib as L


def _p(t):
    return ctypes.c_void_p(t.data_ptr()) if t is not None else None


def upload_weights(named_tensors, dtype: str, device="cuda"):
    """(name, fp32 numpy array, bf16 bits or None) tuples -> dict of CUDA tensors.
    Norm gains (names ending in 'norm') and fast weights ('fast.*') stay fp32;
    other tensors use the configured dtype (bf16 from the given bit patterns)."""
    out = {}
    for name, arr, bits in named_tensors:
        keep_f32 = name.endswith("norm") or name.startswith("fast.") or dtype == "f32"
        if keep_f32:
            out[name] = torch.from_numpy(np.ascontiguousarray(arr, dtype=np.float32)).to(device)
        else:
            if bits is None:
                raise ValueError(f"{name}: bf16 bit patterns required")
            out[name] = torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).to(device).view(torch.bfloat16)
    return out


class Context:
    """One TTT prefill context (ttt_init ... ttt_free)."""

    def __init__(self, cfg, weights: dict, eta=None, k=None, b=None, n_updated=None, stream=None):
        self.cfg = cfg
        self.k = cfg.k if k is None else k
        self.b = cfg.b if b is None else b
        self.eta = cfg.eta if eta is None else eta
        self.n_updated = cfg.n_updated if n_updated is None else n_updated
        self.weights = weights
        self.stream = torch.cuda.current_stream() if stream is None else stream
        self.dtype = L.TTT_BF16 if cfg.dtype == "bf16" else L.TTT_F32
        c = L.ttt_config(cfg.n_layers, cfg.d_model, cfg.n_heads, cfg.head_dim, cfg.d_ff, cfg.vocab, cfg.norm_eps,
                         cfg.rope_theta, self.dtype)
        Lw = cfg.n_layers
        layers = (L.ttt_layer_weights * Lw)()
        for l in range(Lw):
            p = f"layers.{l}."
            layers[l] = L.ttt_layer_weights(*[_p(weights[p + n]) for n in (
                "attn_norm", "wq", "wk", "wv", "wo", "q_norm", "k_norm", "mlp_norm", "w_gate", "w_up", "w_down")])
        fast = (L.ttt_fast_weights * self.n_updated)()
        for i in range(self.n_updated):
            l = Lw - self.n_updated + i
            fast[i] = L.ttt_fast_weights(*[_p(weights[f"fast.{l}.{n}"]) for n in ("w_gate", "w_up", "w_down")])
        w = L.ttt_weights(_p(weights["embed"]), layers, fast, _p(weights["final_norm"]), _p(weights["lm_head"]))
        self._keep = (c, layers, fast, w)
        h = ctypes.c_void_p()
        rc = L.lib().ttt_init(ctypes.byref(c), ctypes.byref(w), self.eta, self.k, self.b, self.n_updated,
                              ctypes.c_void_p(self.stream.cuda_stream), ctypes.byref(h))
        L.check(rc)
        self.h = h

    def fast_out_buffers(self):
        cfg = self.cfg
        f, d = cfg.d_ff, cfg.d_model
        bufs = []
        for _ in range(self.n_updated):
            bufs += [torch.empty(f, d, device="cuda"), torch.empty(f, d, device="cuda"),
                     torch.empty(d, f, device="cuda")]
        return bufs

    def prefill(self, tokens, losses=None, fast_out=None, sync=True):
        """tokens: int32 CUDA tensor [T].  Returns (losses [T] fp32, fast_out list)."""
        T = tokens.numel()
        if losses is None:
            losses = torch.empty(T, device="cuda", dtype=torch.float32)
        arr = None
        if fast_out is not None:
            arr = (ctypes.c_void_p * len(fast_out))(*[t.data_ptr() for t in fast_out])
        rc = L.lib().ttt_prefill(self.h, _p(tokens), T, _p(losses), arr)
        L.check(rc, self.h)
        if sync:
            self.sync()
        return losses, fast_out

    def decode_step(self, out=None, sync=True):
        """ttt_decode_step: one greedy token (int32 CUDA tensor [1])."""
        if out is None:
            out = torch.empty(1, device="cuda", dtype=torch.int32)
        L.check(L.lib().ttt_decode_step(self.h, _p(out)), self.h)
        if sync:
            self.sync()
        return out

    def decode(self, n, tokens=None, losses=None, sync=True):
        """ttt_decode: n greedy tokens (int32 [n]) and, when `losses` is given
        (fp32 [n]), the loss of the position before each token against it."""
        if tokens is None:
            tokens = torch.empty(n, device="cuda", dtype=torch.int32)
        L.check(L.lib().ttt_decode(self.h, n, _p(tokens), _p(losses)), self.h)
        if sync:
            self.sync()
        return tokens, losses

    def reset(self):
        L.check(L.lib().ttt_reset(self.h), self.h)

    def sync(self):
        L.check(L.lib().ttt_sync(self.h), self.h)

    def launch_count(self):
        return int(L.lib().ttt_launch_count(self.h))

    def timing_enable(self, on=True):
        L.check(L.lib().ttt_timing_enable(self.h, 1 if on else 0), self.h)

    def timing_read(self):
        """{class name: (total_ms, launches, algorithmic flops)} since timing_enable."""
        out = {}
        for kc, name in enumerate(L.KC_NAMES):
            ms, n, fl = ctypes.c_double(), ctypes.c_int64(), ctypes.c_double()
            L.check(L.lib().ttt_timing_read(self.h, kc, ctypes.byref(ms), ctypes.byref(n), ctypes.byref(fl)), self.h)
            out[name] = (ms.value, n.value, fl.value)
        return out

    def close(self):
        if getattr(self, "h", None):
            L.lib().ttt_free(self.h)
            self.h = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    def fast_dict(self, fast_out):
        """Map the flat fast_out list to {layer: {name: tensor}}."""
        Lw = self.cfg.n_layers
        out = {}
        for i in range(self.n_updated):
            l = Lw - self.n_updated + i
            out[l] = {"w_gate": fast_out[3 * i], "w_up": fast_out[3 * i + 1], "w_down": fast_out[3 * i + 2]}
        return out
