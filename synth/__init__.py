"""Seeded synthetic inputs shared by the CUDA path and the CPU oracle.

This module draws token streams and initial weights; it performs none of the
method's arithmetic.  The pages measure on Books/DCLM text with the Llama3
tokenizer (End-to-End Test-Time Training for Long Context, reading notes
§9.1; recipe in the jdon.com write-up, appendix "basic recipe"), which are not
available here.  A Zipf(1.1) token stream with 64-token spans repeated at
log-uniform distances stands in for them, at the same vocabulary size and
sequence lengths.  Weights are N(0, 0.02^2); RMSNorm gains are 1.

The heavy lifting is in ``gen.c`` (SplitMix64 counter-based streams, OpenMP);
it is compiled on first use with gcc.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading
from dataclasses import dataclass, replace

import numpy as np

from .configs import CONFIGS, ModelConfig, get_config  # noqa: F401

_HERE = os.path.dirname(os.path.abspath(__file__))
_SO = os.path.join(_HERE, "_gen.so")
_lib = None
_lock = threading.Lock()

WEIGHT_STD = 0.02
ZIPF_ALPHA = 1.1
SPAN = 64
GAP_LO, GAP_HI = 128, 1024


def build(force: bool = False) -> str:
    """Compile gen.c into _gen.so next to it (gcc, OpenMP)."""
    src = os.path.join(_HERE, "gen.c")
    if force or not os.path.exists(_SO) or os.path.getmtime(_SO) < os.path.getmtime(src):
        tmp = _SO + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", "-O2", "-fopenmp", "-shared", "-fPIC", src, "-o", tmp, "-lm"])
        os.replace(tmp, _SO)
    return _SO


def _load():
    global _lib
    with _lock:
        if _lib is None:
            build()
            lib = ctypes.CDLL(_SO)
            u64, i64, i32 = ctypes.c_uint64, ctypes.c_int64, ctypes.c_int32
            vp = ctypes.c_void_p
            lib.synth_stream_key.restype = u64
            lib.synth_stream_key.argtypes = [u64, u64]
            lib.synth_u64.restype = u64
            lib.synth_u64.argtypes = [u64, u64]
            lib.synth_normal_f32.restype = None
            lib.synth_normal_f32.argtypes = [u64, i64, ctypes.c_double, vp]
            lib.synth_round_bf16.restype = None
            lib.synth_round_bf16.argtypes = [vp, i64, vp, vp]
            lib.synth_tokens.restype = ctypes.c_int
            lib.synth_tokens.argtypes = [u64, i64, i32, ctypes.c_double, i32, i32, i32, vp]
            _lib = lib
    return _lib


def _ptr(a: np.ndarray):
    return ctypes.c_void_p(a.ctypes.data) if a is not None else None


def stream_key(seed: int, stream: int) -> int:
    return int(_load().synth_stream_key(seed & (2**64 - 1), stream & (2**64 - 1)))


def normal(seed: int, stream: int, shape, std: float = WEIGHT_STD) -> np.ndarray:
    """float32 array of N(0, std^2) draws from stream (seed, stream)."""
    out = np.empty(shape, dtype=np.float32)
    _load().synth_normal_f32(stream_key(seed, stream), out.size, float(std), _ptr(out))
    return out


def round_bf16(x: np.ndarray):
    """Round fp32 -> bf16 (nearest-even).  Returns (uint16 bits, rounded fp32)."""
    x = np.ascontiguousarray(x, dtype=np.float32)
    bits = np.empty(x.shape, dtype=np.uint16)
    wide = np.empty(x.shape, dtype=np.float32)
    _load().synth_round_bf16(_ptr(x), x.size, _ptr(bits), _ptr(wide))
    return bits, wide


def tokens(cfg: ModelConfig, T: int | None = None, seed: int | None = None) -> np.ndarray:
    """int32 token stream of length T (default cfg.T) for the config's vocab."""
    T = cfg.T if T is None else T
    seed = cfg.seed if seed is None else seed
    out = np.empty(T, dtype=np.int32)
    rc = _load().synth_tokens(seed, T, cfg.vocab, ZIPF_ALPHA, SPAN, GAP_LO, GAP_HI, _ptr(out))
    if rc != 0:
        raise ValueError("synth_tokens: bad arguments")
    return out


# stream ids: (kind << 32) | layer index
_KIND = {"embed": 1, "wq": 2, "wk": 3, "wv": 4, "wo": 5, "w_gate": 6, "w_up": 7, "w_down": 8,
         "fast_gate": 9, "fast_up": 10, "fast_down": 11, "lm_head": 12}


def _stream(kind: str, layer: int = 0) -> int:
    return (_KIND[kind] << 32) | layer


@dataclass
class Weights:
    """Initial weights as float32 arrays.  For bf16 configs every linear weight
    is already rounded to bf16 (the values both sides use); ``bits`` then holds
    the bf16 bit patterns of the same tensors, keyed like ``arrays``."""

    cfg: ModelConfig
    arrays: dict
    bits: dict


def weight_specs(cfg: ModelConfig):
    """Yield (name, shape, stream or None) in a fixed order.  stream None means a
    norm gain initialised to ones."""
    L, d, f, V, hd = cfg.n_layers, cfg.d_model, cfg.d_ff, cfg.vocab, cfg.head_dim
    yield "embed", (V, d), _stream("embed")
    for l in range(L):
        yield f"layers.{l}.attn_norm", (d,), None
        yield f"layers.{l}.wq", (d, d), _stream("wq", l)
        yield f"layers.{l}.wk", (d, d), _stream("wk", l)
        yield f"layers.{l}.wv", (d, d), _stream("wv", l)
        yield f"layers.{l}.wo", (d, d), _stream("wo", l)
        yield f"layers.{l}.q_norm", (hd,), None
        yield f"layers.{l}.k_norm", (hd,), None
        yield f"layers.{l}.mlp_norm", (d,), None
        yield f"layers.{l}.w_gate", (f, d), _stream("w_gate", l)
        yield f"layers.{l}.w_up", (f, d), _stream("w_up", l)
        yield f"layers.{l}.w_down", (d, f), _stream("w_down", l)
    for i in range(cfg.n_updated):
        l = L - cfg.n_updated + i
        yield f"fast.{l}.w_gate", (f, d), _stream("fast_gate", l)
        yield f"fast.{l}.w_up", (f, d), _stream("fast_up", l)
        yield f"fast.{l}.w_down", (d, f), _stream("fast_down", l)
    yield "final_norm", (d,), None
    yield "lm_head", (V, d), _stream("lm_head")


def iter_weights(cfg: ModelConfig, seed: int | None = None):
    """Yield (name, fp32 array, bf16 bits or None) one tensor at a time."""
    wseed = (cfg.seed if seed is None else seed) + 1
    for name, shape, stream in weight_specs(cfg):
        if stream is None:
            a = np.ones(shape, dtype=np.float32)
            yield name, a, None
            continue
        a = normal(wseed, stream, shape)
        if cfg.dtype == "bf16":
            bits, a = round_bf16(a)
            yield name, a, bits
        else:
            yield name, a, None


def make_weights(cfg: ModelConfig, seed: int | None = None, keep_bits: bool = True) -> Weights:
    arrays, bits = {}, {}
    for name, a, b in iter_weights(cfg, seed):
        arrays[name] = a
        if b is not None and keep_bits:
            bits[name] = b
    return Weights(cfg, arrays, bits)


__all__ = ["CONFIGS", "ModelConfig", "get_config", "tokens", "make_weights", "iter_weights",
           "weight_specs", "normal", "round_bf16", "Weights", "build", "replace"]
