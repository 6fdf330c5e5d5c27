"""torch-tensor wrappers of the op-level entry points (include/ttt_ops.h).
Argument marshalling only."""
from __future__ import annotations

import ctypes

import torch

from . import _lib as L


def _p(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream):
    s = torch.cuda.current_stream() if stream is None else stream
    return ctypes.c_void_p(s.cuda_stream)


def _dtype(t):
    if t.dtype == torch.bfloat16:
        return L.TTT_BF16
    if t.dtype == torch.float32:
        return L.TTT_F32
    raise TypeError(f"unsupported dtype {t.dtype}")


def _epi_args(c=None, c2=None, row_f=None, row_g=None, row_i=None, part_max=None, part_sum=None,
              target_logit=None, part_ld=0, alpha=0.0, col_offset=0, c3=None):
    return L.ttt_epilogue_args(
        _p(c), c.stride(0) if c is not None else 0, _p(c2), c2.stride(0) if c2 is not None else 0,
        _p(row_f), _p(row_g), _p(row_i), _p(part_max), _p(part_sum), _p(target_logit), part_ld, alpha, col_offset,
        _p(c3), c3.stride(0) if c3 is not None else 0)


def gemm(A, B, a_mn, b_mn, epi, c=None, c2=None, row_f=None, row_g=None, row_i=None, part_max=None,
         part_sum=None, target_logit=None, part_ld=0, alpha=0.0, col_offset=0, bn=0, M=None, N=None, K=None,
         c3=None, stream=None):
    """ttt_op_gemm on 2-D tensors in storage order (see ttt_ops.h)."""
    dt = _dtype(A)
    M = (A.shape[1] if a_mn else A.shape[0]) if M is None else M
    K = (A.shape[0] if a_mn else A.shape[1]) if K is None else K
    N = (B.shape[1] if b_mn else B.shape[0]) if N is None else N
    args = _epi_args(c, c2, row_f, row_g, row_i, part_max, part_sum, target_logit, part_ld, alpha, col_offset, c3)
    rc = L.lib().ttt_op_gemm(dt, int(a_mn), int(b_mn), M, N, K, _p(A), A.stride(0), _p(B), B.stride(0), epi,
                             ctypes.byref(args), bn, _stream(stream))
    L.check(rc)


def gemm_split(A, B, a_mn, b_mn, epi, ksplit, workspace, c=None, c2=None, bn=0, stream=None):
    """ttt_op_gemm_split: bf16 GEMM with a deterministic split-K reduction."""
    M = A.shape[1] if a_mn else A.shape[0]
    K = A.shape[0] if a_mn else A.shape[1]
    N = B.shape[1] if b_mn else B.shape[0]
    args = _epi_args(c, c2)
    rc = L.lib().ttt_op_gemm_split(int(a_mn), int(b_mn), M, N, K, _p(A), A.stride(0), _p(B), B.stride(0), epi,
                                   ctypes.byref(args), bn, ksplit, _p(workspace), _stream(stream))
    L.check(rc)


def gemm_dual(A, B, A2, B2, a_mn, b_mn, epi, n_ext=0, ksplit=1, workspace=None, bn=0, stream=None, **epi_kw):
    """ttt_op_gemm_dual: acc = A B^T, plus A2 B2^T on output columns >= n_ext (bf16)."""
    M = A.shape[1] if a_mn else A.shape[0]
    K = A.shape[0] if a_mn else A.shape[1]
    K2 = A2.shape[0] if a_mn else A2.shape[1]
    N = B.shape[1] if b_mn else B.shape[0]
    args = _epi_args(**epi_kw)
    rc = L.lib().ttt_op_gemm_dual(int(a_mn), int(b_mn), M, N, K, _p(A), A.stride(0), _p(B), B.stride(0), K2, _p(A2),
                                  A2.stride(0), _p(B2), B2.stride(0), n_ext, epi, ctypes.byref(args), bn, ksplit,
                                  _p(workspace), _stream(stream))
    L.check(rc)


def gemm_plan(M, N, K, epi):
    """ttt_op_gemm_plan: (split count, tile width) the prefill uses."""
    bn = ctypes.c_int32(0)
    S = int(L.lib().ttt_op_gemm_plan(M, N, K, epi, ctypes.byref(bn)))
    return S, int(bn.value)


def gemm_ce_tiles(dtype_is_bf16, M, N, bn=0):
    return int(L.lib().ttt_op_gemm_ce_tiles(L.TTT_BF16 if dtype_is_bf16 else L.TTT_F32, M, N, bn))


def sync(stream=None):
    L.check(L.lib().ttt_op_sync(_stream(stream)))


def swa_forward(q, k_ring, v_ring, n_heads, head_dim, q_pos0, window, o, lse, force_simt=False, stream=None,
                q_norm_max=0.0, k_norm_max=0.0, exp_poly=None):
    """ttt_op_swa_forward; q/o [n, H*hd], rings [R, H*hd], lse [H, n].
    q_norm_max, k_norm_max: bounds on the row norms of q and k (0 = unknown;
    both known: the fixed-shift tensor-core forward); exp_poly: its
    polynomial share of the exponentials (0, 2 or 4 of 8; None = default)."""
    flags = 1 if force_simt else 0
    if exp_poly is not None:
        flags |= ((exp_poly + 1) & 15) << 4
    rc = L.lib().ttt_op_swa_forward(_dtype(q), n_heads, head_dim, q.shape[0], q_pos0, window, _p(q), q.stride(0),
                                    _p(k_ring), _p(v_ring), k_ring.shape[0], _p(o), o.stride(0), _p(lse),
                                    float(q_norm_max), float(k_norm_max), flags, _stream(stream))
    L.check(rc)


def swa_backward(q, k_ring, v_ring, n_heads, head_dim, q_pos0, window, o, lse, dout, dq, dk, dv, D,
                 force_simt=False, stream=None):
    """ttt_op_swa_backward; dk/dv rows are the keys at q_pos0 .. q_pos0+n-1."""
    rc = L.lib().ttt_op_swa_backward(_dtype(q), n_heads, head_dim, q.shape[0], q_pos0, window, _p(q), q.stride(0),
                                     _p(k_ring), _p(v_ring), k_ring.shape[0], _p(o), o.stride(0), _p(lse), _p(dout),
                                     dout.stride(0), _p(dq), dq.stride(0), _p(dk), _p(dv), dk.stride(0), _p(D),
                                     1 if force_simt else 0, _stream(stream))
    L.check(rc)


def watchdog_selftest(stream=None):
    """Launch the bounded-wait self-test; ops.sync() afterwards must raise TTT_ERR_TIMEOUT."""
    L.check(L.lib().ttt_op_watchdog_selftest(_stream(stream)))


def swa_backward_noalloc(q, k_ring, v_ring, n_heads, head_dim, q_pos0, window, o, lse, dout, dq, dk, dv,
                         stream=None):
    """ttt_op_swa_backward_noalloc: like swa_backward, with the library's own
    fixed work array instead of caller scratch (no device allocation)."""
    rc = L.lib().ttt_op_swa_backward_noalloc(_dtype(q), n_heads, head_dim, q.shape[0], q_pos0, window, _p(q),
                                             q.stride(0), _p(k_ring), _p(v_ring), k_ring.shape[0], _p(o),
                                             o.stride(0), _p(lse), _p(dout), dout.stride(0), _p(dq), dq.stride(0),
                                             _p(dk), _p(dv), dk.stride(0), _stream(stream))
    L.check(rc)


def rmsnorm(x, g, eps, y, rstd, stream=None):
    """ttt_op_rmsnorm: x fp32 [n, d] -> y bf16 [n, d], rstd fp32 [n]."""
    n, d = x.shape
    L.check(L.lib().ttt_op_rmsnorm(n, d, _p(x), x.stride(0), _p(g), eps, _p(y), y.stride(0), _p(rstd),
                                   _stream(stream)))


def qknorm_rope(qkv, p0, n_heads, head_dim, eps, theta, gq, gk, qout, kring, vring, rq, rk, tab, stream=None):
    """ttt_op_qknorm_rope: qkv bf16 [n, 3*H*hd] at positions p0.. -> qout, ring slots, rq/rk [n, H]."""
    n = qkv.shape[0]
    L.check(L.lib().ttt_op_qknorm_rope(n, p0, n_heads, head_dim, eps, theta, _p(qkv), qkv.stride(0), _p(gq), _p(gk),
                                       _p(qout), qout.stride(0), _p(kring), _p(vring), kring.shape[0], _p(rq),
                                       _p(rk), _p(tab), _stream(stream)))


def swiglu_bwd(da, gu, dgu, stream=None):
    """ttt_op_swiglu_bwd: da [n, F], gu/dgu [n, 2F] interleaved in (gate 64 | up 64) blocks (bf16)."""
    n, nfeat = da.shape
    L.check(L.lib().ttt_op_swiglu_bwd(n, nfeat, _p(da), da.stride(0), _p(gu), gu.stride(0), _p(dgu), dgu.stride(0),
                                      _stream(stream)))


def gemv(epi, w, x, out, res=None, raw=None, lse=None, part=None, stream=None):
    """ttt_op_gemv: y = w x (bf16 w [n, k], x [k]) with epilogue 0 store, 1 add, 2 SwiGLU, 3 greedy pick."""
    n, k = w.shape
    L.check(L.lib().ttt_op_gemv(epi, n, k, _p(w), w.stride(0), _p(x), _p(out), _p(res), _p(raw), _p(lse), _p(part),
                                _stream(stream)))


def attn_decode(q, kring, vring, n_heads, head_dim, p, window, o, lse, ws, stream=None):
    """ttt_op_attn_decode: one query per head (bf16 [H*hd]) over the window of the rings."""
    L.check(L.lib().ttt_op_attn_decode(n_heads, head_dim, p, window, _p(q), _p(kring), _p(vring), kring.shape[0],
                                       _p(o), _p(lse), _p(ws), _stream(stream)))


def meta_grad_work(n_chunks, b, d, f, vocab):
    """ttt_op_meta_grad_work: floats of scratch ttt_op_meta_grad needs."""
    n = L.lib().ttt_op_meta_grad_work(n_chunks, b, d, f, vocab)
    if n < 0:
        raise ValueError("meta_grad_work: sizes must be >= 1")
    return n


def meta_grad(h, r, targets, w_gate, w_up, w_down, g_final, w_head, eps, eta, b, d_gate, d_up, d_down,
              losses=None, work=None, stream=None):
    """ttt_op_meta_grad: dL/dW^(0) of the adapted loss over len(targets) / b
    chunks into d_gate, d_up, d_down (fp32, shaped like the weights); the
    per-row losses along the inner loop into ``losses`` when given.  ``work``
    (fp32) is allocated here when not given."""
    rows, d = h.shape
    f = w_gate.shape[0]
    V = w_head.shape[0]
    n_chunks = rows // b
    need = meta_grad_work(n_chunks, b, d, f, V)
    if work is None:
        work = torch.empty(need, dtype=torch.float32, device=h.device)
    L.check(L.lib().ttt_op_meta_grad(n_chunks, b, d, f, V, _p(h), _p(r), _p(targets), _p(w_gate), _p(w_up),
                                     _p(w_down), _p(g_final), _p(w_head), eps, eta, _p(d_gate), _p(d_up),
                                     _p(d_down), _p(losses), _p(work), work.numel(), _stream(stream)))
    return work
