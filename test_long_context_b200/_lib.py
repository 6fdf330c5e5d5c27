"""ctypes binding of libttt_b200.so: the C ABI of include/ttt.h and
include/ttt_ops.h with the same names.  Argument marshalling only; every
step of the computation runs in the CUDA library.  Loading fails loudly when
the library has not been built."""
from __future__ import annotations

import ctypes
import os

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libttt_b200.so")

TTT_OK = 0
TTT_ERR_INVALID_ARG = -1
TTT_ERR_STATE = -2
TTT_ERR_OOM = -3
TTT_ERR_CUDA = -4
TTT_ERR_TIMEOUT = -5
TTT_ERR_UNSUPPORTED = -6
TTT_F32 = 0
TTT_BF16 = 1

KC_GEMM, KC_ATTN_FWD, KC_ATTN_BWD, KC_OTHER, KC_NORM, KC_ROPE, KC_DECODE = range(7)
KC_NAMES = ("gemm", "attn_fwd", "attn_bwd", "other", "norm", "rope", "decode")
EPI_STORE_F32, EPI_STORE_BF16, EPI_ADD_F32, EPI_SWIGLU, EPI_CE_FWD, EPI_CE_BWD, EPI_SGD = range(7)

c_i32, c_i64, c_f32, c_vp = ctypes.c_int32, ctypes.c_int64, ctypes.c_float, ctypes.c_void_p


class ttt_config(ctypes.Structure):
    _fields_ = [("n_layers", c_i32), ("d_model", c_i32), ("n_heads", c_i32), ("head_dim", c_i32),
                ("d_ff", c_i32), ("vocab", c_i32), ("norm_eps", c_f32), ("rope_theta", c_f32), ("dtype", c_i32)]


class ttt_layer_weights(ctypes.Structure):
    _fields_ = [(n, c_vp) for n in ("attn_norm", "wq", "wk", "wv", "wo", "q_norm", "k_norm", "mlp_norm",
                                    "w_gate", "w_up", "w_down")]


class ttt_fast_weights(ctypes.Structure):
    _fields_ = [(n, c_vp) for n in ("w_gate", "w_up", "w_down")]


class ttt_weights(ctypes.Structure):
    _fields_ = [("embed", c_vp), ("layers", ctypes.POINTER(ttt_layer_weights)),
                ("fast", ctypes.POINTER(ttt_fast_weights)), ("final_norm", c_vp), ("lm_head", c_vp)]


class ttt_epilogue_args(ctypes.Structure):
    _fields_ = [("c", c_vp), ("ldc", c_i64), ("c2", c_vp), ("ldc2", c_i64), ("row_f", c_vp), ("row_g", c_vp),
                ("row_i", c_vp), ("part_max", c_vp), ("part_sum", c_vp), ("target_logit", c_vp),
                ("part_ld", c_i64), ("alpha", c_f32), ("col_offset", c_i64), ("c3", c_vp), ("ldc3", c_i64)]


_lib = None


def lib():
    """The loaded CUDA library (raises if it was not built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"CUDA library not built: {LIB_PATH} (run python -m test_long_context_b200.build)")
        L = ctypes.CDLL(LIB_PATH)
        sig = {
            "ttt_init": (c_i32, [ctypes.POINTER(ttt_config), ctypes.POINTER(ttt_weights), c_f32, c_i32, c_i32,
                                 c_i32, c_vp, ctypes.POINTER(c_vp)]),
            "ttt_prefill": (c_i32, [c_vp, c_vp, c_i64, c_vp, ctypes.POINTER(c_vp)]),
            "ttt_decode_step": (c_i32, [c_vp, c_vp]),
            "ttt_decode": (c_i32, [c_vp, c_i64, c_vp, c_vp]),
            "ttt_reset": (c_i32, [c_vp]),
            "ttt_sync": (c_i32, [c_vp]),
            "ttt_last_error": (ctypes.c_char_p, [c_vp]),
            "ttt_free": (None, [c_vp]),
            "ttt_launch_count": (c_i64, [c_vp]),
            "ttt_timing_enable": (c_i32, [c_vp, c_i32]),
            "ttt_timing_read": (c_i32, [c_vp, c_i32, ctypes.POINTER(ctypes.c_double), ctypes.POINTER(c_i64),
                                        ctypes.POINTER(ctypes.c_double)]),
            "ttt_op_gemm": (c_i32, [c_i32, c_i32, c_i32, c_i64, c_i64, c_i64, c_vp, c_i64, c_vp, c_i64, c_i32,
                                    ctypes.POINTER(ttt_epilogue_args), c_i32, c_vp]),
            "ttt_op_gemm_ce_tiles": (c_i64, [c_i32, c_i64, c_i64, c_i32]),
            "ttt_op_gemm_dual": (c_i32, [c_i32, c_i32, c_i64, c_i64, c_i64, c_vp, c_i64, c_vp, c_i64, c_i64, c_vp,
                                         c_i64, c_vp, c_i64, c_i64, c_i32, ctypes.POINTER(ttt_epilogue_args), c_i32,
                                         c_i32, c_vp, c_vp]),
            "ttt_op_gemm_split": (c_i32, [c_i32, c_i32, c_i64, c_i64, c_i64, c_vp, c_i64, c_vp, c_i64, c_i32,
                                          ctypes.POINTER(ttt_epilogue_args), c_i32, c_i32, c_vp, c_vp]),
            "ttt_op_sync": (c_i32, [c_vp]),
            "ttt_op_gemm_plan": (c_i64, [c_i64, c_i64, c_i64, c_i32, ctypes.POINTER(c_i32)]),
            "ttt_op_watchdog_selftest": (c_i32, [c_vp]),
            "ttt_op_swa_backward_noalloc": (c_i32, [c_i32, c_i32, c_i32, c_i64, c_i64, c_i32, c_vp, c_i64, c_vp,
                                                    c_vp, c_i64, c_vp, c_i64, c_vp, c_vp, c_i64, c_vp, c_i64, c_vp,
                                                    c_vp, c_i64, c_vp]),
            "ttt_op_swa_forward": (c_i32, [c_i32, c_i32, c_i32, c_i64, c_i64, c_i32, c_vp, c_i64, c_vp, c_vp, c_i64,
                                           c_vp, c_i64, c_vp, c_f32, c_f32, c_i32, c_vp]),
            "ttt_op_swa_backward": (c_i32, [c_i32, c_i32, c_i32, c_i64, c_i64, c_i32, c_vp, c_i64, c_vp, c_vp,
                                            c_i64, c_vp, c_i64, c_vp, c_vp, c_i64, c_vp, c_i64, c_vp, c_vp, c_i64,
                                            c_vp, c_i32, c_vp]),
            "ttt_op_rmsnorm": (c_i32, [c_i64, c_i32, c_vp, c_i64, c_vp, c_f32, c_vp, c_i64, c_vp, c_vp]),
            "ttt_op_qknorm_rope": (c_i32, [c_i64, c_i64, c_i32, c_i32, c_f32, c_f32, c_vp, c_i64, c_vp, c_vp, c_vp,
                                           c_i64, c_vp, c_vp, c_i64, c_vp, c_vp, c_vp, c_vp]),
            "ttt_op_swiglu_bwd": (c_i32, [c_i64, c_i64, c_vp, c_i64, c_vp, c_i64, c_vp, c_i64, c_vp]),
            "ttt_op_gemv": (c_i32, [c_i32, c_i64, c_i64, c_vp, c_i64, c_vp, c_vp, c_vp, c_vp, c_vp, c_vp, c_vp]),
            "ttt_op_attn_decode": (c_i32, [c_i32, c_i32, c_i64, c_i32, c_vp, c_vp, c_vp, c_i64, c_vp, c_vp, c_vp,
                                           c_vp]),
            "ttt_op_meta_grad_work": (c_i64, [c_i64, c_i64, c_i32, c_i32, c_i64]),
            "ttt_op_meta_grad": (c_i32, [c_i64, c_i64, c_i32, c_i32, c_i64, c_vp, c_vp, c_vp, c_vp, c_vp, c_vp, c_vp,
                                         c_vp, c_f32, c_f32, c_vp, c_vp, c_vp, c_vp, c_vp, c_i64, c_vp]),
        }
        for name, (res, args) in sig.items():
            if hasattr(L, name):
                fn = getattr(L, name)
                fn.restype = res
                fn.argtypes = args
        _lib = L
    return _lib


class TTTError(RuntimeError):
    def __init__(self, code, msg):
        super().__init__(f"{msg} (code {code})")
        self.code = code


def check(rc, ctx=None):
    if rc != TTT_OK:
        msg = lib().ttt_last_error(ctx)
        raise TTTError(rc, msg.decode() if msg else "unknown error")
    return rc


def exported_symbols():
    """Names of the ttt_* entry points the loaded library exports."""
    L = lib()
    names = []
    for n in ("ttt_init", "ttt_prefill", "ttt_decode_step", "ttt_decode", "ttt_reset", "ttt_sync", "ttt_last_error", "ttt_free",
              "ttt_launch_count", "ttt_timing_enable", "ttt_timing_read", "ttt_op_gemm", "ttt_op_gemm_split", "ttt_op_gemm_dual", "ttt_op_gemm_ce_tiles", "ttt_op_gemm_plan", "ttt_op_sync", "ttt_op_swa_forward",
              "ttt_op_swa_backward", "ttt_op_watchdog_selftest", "ttt_op_rmsnorm", "ttt_op_qknorm_rope",
              "ttt_op_swiglu_bwd", "ttt_op_gemv", "ttt_op_attn_decode",
              "ttt_op_swa_backward_noalloc", "ttt_op_meta_grad_work", "ttt_op_meta_grad"):
        if hasattr(L, n):
            names.append(n)
    return names
