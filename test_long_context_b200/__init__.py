"""B200-native (sm_100a) TTT-E2E prefill: the CUDA library and its binding.

The computation lives in libttt_b200.so (include/ttt.h, include/ttt_ops.h);
this package only marshals arguments.  ``Context`` wraps ttt_init /
ttt_prefill / ttt_reset for torch tensors; ``ops`` exposes the op-level
entry points used by the kernel tests."""
from ._lib import TTTError, check, lib  # noqa: F401
