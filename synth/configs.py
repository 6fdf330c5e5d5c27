"""Model and sequence configurations of the TTT-E2E prefill workloads.

Model shapes follow the recipe in the jdon.com write-up (section "参数细节",
125M / 760M / 2.7B rows: layers, width, heads) with the SwiGLU hidden sizes,
vocabulary and head dims of the workload definitions; window k = 8K, chunk
b = 1K and "update the last quarter of the MLP blocks" come from the same
section (k, b, fraction).  The inner learning rate is 1e-2 for every config:
only the tiny config states it, and the others say "same distributions".
"""
from __future__ import annotations

from dataclasses import dataclass, replace


@dataclass(frozen=True)
class ModelConfig:
    name: str
    n_layers: int
    d_model: int
    n_heads: int
    head_dim: int
    d_ff: int
    vocab: int
    n_updated: int  # blocks L-n_updated .. L-1 carry a fast MLP
    T: int          # tokens per sequence
    k: int          # attention window (keys per query, self included)
    b: int          # TTT chunk size
    eta: float      # inner SGD learning rate
    dtype: str      # "f32" or "bf16"
    seed: int
    norm_eps: float = 1e-5
    rope_theta: float = 10000.0

    def with_(self, **kw) -> "ModelConfig":
        return replace(self, **kw)

    @property
    def n_chunks(self) -> int:
        return -(-self.T // self.b)


_SEED0 = 0x7E2E0000

CONFIGS = {
    "tiny": ModelConfig("tiny", 4, 128, 4, 32, 512, 1024, 1, 4096, 1024, 256, 1e-2, "f32", _SEED0 + 0),
    "125m": ModelConfig("125m", 12, 768, 12, 64, 2048, 128256, 3, 8192, 8192, 1024, 1e-2, "bf16", _SEED0 + 1),
    "760m": ModelConfig("760m", 24, 1536, 16, 96, 4096, 128256, 6, 32768, 8192, 1024, 1e-2, "bf16", _SEED0 + 2),
    "2.7b": ModelConfig("2.7b", 32, 2560, 32, 80, 6912, 128256, 8, 131072, 8192, 1024, 1e-2, "bf16", _SEED0 + 3),
}


def get_config(name: str, **overrides) -> ModelConfig:
    cfg = CONFIGS[name]
    return replace(cfg, **overrides) if overrides else cfg
