"""CPU oracle of the TTT-E2E prefill loop — test infrastructure only.

Imported by tests/, __graft_entry__.smoke() and bench.py's CPU-baseline and
reference legs; never by the CUDA library or its Python binding."""
from .ttt_oracle import (Model, Result, State, backward_chunk, forward_chunk, init_fast,  # noqa: F401
                         prefill, static_losses, window_pairs)
