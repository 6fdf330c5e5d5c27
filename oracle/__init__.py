"""CPU oracle of the TTT-E2E prefill loop — test infrastructure only.

Imported by tests/, __graft_entry__.smoke() and bench.py's CPU-baseline and
reference legs; never by the CUDA library or its Python binding."""
from .ttt_oracle import (DecodeResult, Model, Result, State, backward_chunk, decode, forward_chunk,  # noqa: F401
                         init_fast, prefill, static_losses, window_pairs)
