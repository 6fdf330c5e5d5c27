"""CPU-side checks of the C ABI: the library loads and exports every symbol
the headers declare (no compute calls without a GPU)."""
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared():
    names = set()
    for h in ("ttt.h", "ttt_ops.h"):
        with open(os.path.join(ROOT, "include", h)) as fh:
            src = fh.read()
        src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
        names |= set(re.findall(r"\b(ttt_[a-z_0-9]+)\s*\(", src))
    return names


def test_library_exports_every_declared_symbol():
    from test_long_context_b200 import _lib
    from test_long_context_b200.build import build
    build()
    L = _lib.lib()
    missing = [n for n in sorted(_declared()) if not hasattr(L, n)]
    assert not missing, missing
    assert {"ttt_init", "ttt_prefill", "ttt_decode_step", "ttt_reset", "ttt_sync", "ttt_free"} <= _declared()


def test_init_rejects_bad_arguments_without_gpu():
    """Argument validation happens on the host before any device call."""
    import ctypes
    from test_long_context_b200 import _lib as L
    lib = L.lib()
    h = ctypes.c_void_p()
    assert lib.ttt_init(None, None, 0.01, 8, 4, 1, None, ctypes.byref(h)) == L.TTT_ERR_INVALID_ARG
    cfg = L.ttt_config(2, 96, 2, 48, 128, 64, 1e-5, 10000.0, L.TTT_F32)  # head_dim 48 unsupported
    w = L.ttt_weights()
    rc = lib.ttt_init(ctypes.byref(cfg), ctypes.byref(w), 0.01, 8, 4, 1, None, ctypes.byref(h))
    assert rc in (L.TTT_ERR_INVALID_ARG, L.TTT_ERR_UNSUPPORTED)
    cfg = L.ttt_config(2, 64, 2, 32, 128, 64, 1e-5, 10000.0, L.TTT_F32)
    rc = lib.ttt_init(ctypes.byref(cfg), ctypes.byref(w), float("nan"), 8, 4, 1, None, ctypes.byref(h))
    assert rc == L.TTT_ERR_INVALID_ARG
    rc = lib.ttt_init(ctypes.byref(cfg), ctypes.byref(w), 0.01, 8, 4, 3, None, ctypes.byref(h))
    assert rc == L.TTT_ERR_INVALID_ARG  # n_updated > n_layers
    assert h.value is None
    assert lib.ttt_prefill(None, None, 1, None, None) == L.TTT_ERR_INVALID_ARG
    assert b"NULL" in lib.ttt_last_error(None)


def test_python_binding_has_no_compute():
    """The binding marshals arguments only: no numpy/torch math on the data path."""
    for f in ("context.py", "ops.py", "_lib.py"):
        with open(os.path.join(ROOT, "test_long_context_b200", f)) as fh:
            src = fh.read()
        assert "import oracle" not in src and "from oracle" not in src


def test_meta_grad_validates_on_the_host():
    """ttt_op_meta_grad checks its arguments before any device call; its
    scratch size follows from the shapes alone."""
    from test_long_context_b200 import _lib as L
    lib = L.lib()
    N, b, d, f, V = 3, 40, 64, 96, 500
    P = 3 * d * f
    assert lib.ttt_op_meta_grad_work(N, b, d, f, V) == N * P + 3 * P + 12 * b * f + 8 * b * d + 3 * b + 3 * b * V + 1
    assert lib.ttt_op_meta_grad_work(0, b, d, f, V) == -1
    fake = 256  # never dereferenced: every call below fails validation first
    args = [fake] * 8
    rc = lib.ttt_op_meta_grad(N, b, d, f, V, *args, 1e-5, 0.5, fake, fake, fake, None, None, 0, None)
    assert rc == L.TTT_ERR_INVALID_ARG  # no work array
    rc = lib.ttt_op_meta_grad(N, b, d, f, V, *args, 1e-5, 0.5, fake, fake, fake, None, fake,
                              lib.ttt_op_meta_grad_work(N, b, d, f, V) - 1, None)
    assert rc == L.TTT_ERR_INVALID_ARG and b"work" in lib.ttt_last_error(None)
    rc = lib.ttt_op_meta_grad(N, b, d, f, V, *args, 1e-5, float("nan"), fake, fake, fake, None, fake, 1 << 40, None)
    assert rc == L.TTT_ERR_INVALID_ARG
    rc = lib.ttt_op_meta_grad(N, b, d, f, V, *args, 0.0, 0.5, fake, fake, fake, None, fake, 1 << 40, None)
    assert rc == L.TTT_ERR_INVALID_ARG
