"""CPU oracle of the outer-loop meta-gradient — TEST INFRASTRUCTURE ONLY.

Only ``tests/``, ``__graft_entry__.smoke()`` and the ``cpu_baseline`` /
``--impl reference`` legs of ``bench.py`` may import this module.  The CUDA
library never calls it and shares no code with it.

What it computes (End-to-End Test-Time Training for Long Context; reading
notes by Zhongzhu Zhou, §4 "元梯度究竟多出了什么"):

  * the inner loop over N chunks takes one SGD step per chunk,
    W^(c+1) = W^(c) - eta * grad A_c(W^(c))                        (eq. (5), U(W));
  * the outer loss is the mean chunk loss along that trajectory,
    L(W^(0)) = (1/N) * sum_c A_c(W^(c))                             (eq. (4), L_adapt, by chunks);
  * its gradient with respect to the starting point is
    grad L = (1/N) * sum_c J_c^T grad A_c(W^(c)),
    J_0 = I, J_(c+1) = (I - eta H_c) J_c, H_c = Hessian of A_c at W^(c)  (eq. (7)),
    which needs only Hessian-vector products (eq. (6): (I - eta H)^T v,
    H symmetric).  ``meta_grad`` evaluates the sum backwards:
    u = grad A_(N-1) / N;  u <- u - eta H_c u + grad A_c / N  for c = N-2 .. 0.

The chunk loss A is that of the model whose LAST block alone carries fast
weights (n_u = 1): the block's fast SwiGLU MLP reads the block's MLP-norm
output h and adds to the residual r (the residual after attention plus the
static MLP), then the final RMSNorm, the LM head and the next-token
cross-entropy (mean over the chunk's targets, eq. (9)):

    A(W) = mean_valid CE(RMSNorm_f(r + SwiGLU(h; W)) head^T, target).

Nothing after that MLP feeds an attention layer, so h and r of every chunk
are independent of W: eq. (7) is then exact (no path through the static
parameters or through cached keys and values, which the pages' derivation
leaves out).  The Hessian-vector product is the directional derivative of
the hand-derived gradient (forward mode over the backward), written out
step by step; the pages only say that automatic differentiation provides
it (§4.1, the paragraph after eq. (6)).

All arithmetic is float64.
"""
from __future__ import annotations

import numpy as np

from .ttt_oracle import log_softmax_ce, rmsnorm, rmsnorm_bwd, sigmoid

F = np.float64


# ----------------------------------------------------------------------------
# one chunk of the last block's fast MLP


def _silu_derivs(g):
    """silu(g) = g s(g), its first and second derivatives (s = sigmoid)."""
    s = sigmoid(g)
    d1 = s * (1.0 + g * (1.0 - s))
    d2 = s * (1.0 - s) * (2.0 + g * (1.0 - 2.0 * s))
    return g * s, d1, d2


def chunk_forward(h, r, tgt, W, gf, head, eps):
    """Forward of one chunk: per-row loss (NaN without a target) and A."""
    wg, wu, wd = W
    G = h @ wg.T
    U = h @ wu.T
    sl, d1, d2 = _silu_derivs(G)
    a = sl * U
    x = r + a @ wd.T
    n_, rr = rmsnorm(x, gf, eps)
    z = n_ @ head.T
    valid = tgt >= 0
    loss = np.full(len(tgt), np.nan)
    nc = int(valid.sum())
    P = np.zeros_like(z)
    if nc:
        lv, pv, _ = log_softmax_ce(z[valid], tgt[valid])
        loss[valid] = lv
        P[valid] = pv
    A = float(np.nansum(loss) / nc) if nc else 0.0
    return dict(h=h, G=G, U=U, sl=sl, d1=d1, d2=d2, a=a, x=x, rr=rr, P=P, valid=valid, tgt=tgt, nc=nc,
                loss=loss, A=A)


def chunk_grad(fw, W, gf, head):
    """grad A with respect to (w_gate, w_up, w_down), and the intermediate
    adjoints the Hessian-vector product reuses."""
    wg, wu, wd = W
    n = len(fw["tgt"])
    w = 1.0 / fw["nc"] if fw["nc"] else 0.0
    dz = fw["P"].copy()
    rows = np.nonzero(fw["valid"])[0]
    dz[rows, fw["tgt"][rows]] -= 1.0
    dz *= w
    dn = dz @ head
    dx = rmsnorm_bwd(fw["x"], fw["rr"], gf, dn)
    dwd = dx.T @ fw["a"]
    da = dx @ wd
    dG = da * fw["U"] * fw["d1"]
    dU = da * fw["sl"]
    grads = (dG.T @ fw["h"], dU.T @ fw["h"], dwd)
    return grads, dict(dn=dn, dx=dx, da=da, w=w, n=n)


def chunk_hvp(fw, bw, W, gf, head, eps, V):
    """H V: the derivative of chunk_grad along V = (v_gate, v_up, v_down)
    (forward-mode tangent of every step of the forward and the backward)."""
    wg, wu, wd = W
    vg, vu, vd = V
    h, G, U, sl, d1, d2, a, x, rr = (fw[k] for k in ("h", "G", "U", "sl", "d1", "d2", "a", "x", "rr"))
    dn, dx, da, w = bw["dn"], bw["dx"], bw["da"], bw["w"]
    # forward tangents
    Gt = h @ vg.T
    Ut = h @ vu.T
    at = d1 * Gt * U + sl * Ut
    xt = at @ wd.T + a @ vd.T
    dd = x.shape[-1]
    rrt = -rr ** 3 * np.sum(x * xt, axis=-1, keepdims=True) / dd
    nt = gf * (xt * rr + x * rrt)
    zt = nt @ head.T
    # cross-entropy: dz = w (P - onehot); its tangent is w P (zt - <P, zt>)
    P = fw["P"]
    c = np.sum(P * zt, axis=-1, keepdims=True)
    dzt = w * P * (zt - c)
    dzt[~fw["valid"]] = 0.0
    dnt = dzt @ head
    # RMSNorm backward dx = rr q - rr^3 x m, q = gf dn, m = mean(x q); its tangent
    q = gf * dn
    qt = gf * dnt
    m = np.sum(x * q, axis=-1, keepdims=True) / dd
    mt = np.sum(xt * q + x * qt, axis=-1, keepdims=True) / dd
    dxt = rrt * q + rr * qt - 3.0 * rr ** 2 * rrt * x * m - rr ** 3 * xt * m - rr ** 3 * x * mt
    # fast MLP backward and its tangent
    dwdt = dxt.T @ a + dx.T @ at
    dat = dxt @ wd + dx @ vd
    dGt = dat * U * d1 + da * Ut * d1 + da * U * d2 * Gt
    dUt = dat * sl + da * d1 * Gt
    return (dGt.T @ h, dUt.T @ h, dwdt)


# ----------------------------------------------------------------------------
# the outer-loop recursion (eq. (7)), for any chunk loss


def _axpy(y, alpha, x):
    return tuple(yi + alpha * xi for yi, xi in zip(y, x))


def inner_loop(n_chunks, W0, eta, loss_grad):
    """W^(c+1) = W^(c) - eta grad A_c(W^(c)) (eq. (5)); returns the
    trajectory W^(0..N-1) and the chunk losses A_c(W^(c))."""
    W = tuple(np.array(w, dtype=F) for w in W0)
    traj, losses = [], []
    for c in range(n_chunks):
        traj.append(W)
        A, g = loss_grad(c, W)
        losses.append(A)
        W = _axpy(W, -eta, g)
    return traj, losses


def meta_grad(n_chunks, W0, eta, loss_grad, hvp):
    """grad of L(W^(0)) = (1/N) sum_c A_c(W^(c)) by eq. (7), evaluated from
    the last chunk backwards with Hessian-vector products (eq. (6)).
    ``loss_grad(c, W) -> (A_c, grad)``; ``hvp(c, W, v) -> H_c v``."""
    traj, losses = inner_loop(n_chunks, W0, eta, loss_grad)
    N = n_chunks
    u = None
    for c in range(N - 1, -1, -1):
        _, g = loss_grad(c, traj[c])
        if u is None:
            u = tuple(gi / N for gi in g)
        else:
            Hu = hvp(c, traj[c], u)
            u = _axpy(_axpy(u, -eta, Hu), 1.0 / N, g)
    return u, float(np.mean(losses)), losses


# ----------------------------------------------------------------------------
# the last block's fast MLP over a sequence of chunks


def _chunk_rows(c, b):
    return slice(c * b, (c + 1) * b)


def meta_grad_top_mlp(h, r, tgt, W0, gf, head, eta, eps, b):
    """eq. (7) for the chunk loss of the module docstring.  h, r: [N*b, d];
    tgt: [N*b] next-token ids (-1: no target).  Returns (grad, L, per-row
    losses along the trajectory)."""
    h, r, gf, head = (np.asarray(t, dtype=F) for t in (h, r, gf, head))
    tgt = np.asarray(tgt, dtype=np.int64)
    N = len(tgt) // b
    rows_loss = np.full(N * b, np.nan)

    def loss_grad(c, W):
        s = _chunk_rows(c, b)
        fw = chunk_forward(h[s], r[s], tgt[s], W, gf, head, eps)
        rows_loss[s] = fw["loss"]
        g, _ = chunk_grad(fw, W, gf, head)
        return fw["A"], g

    def hvp(c, W, v):
        s = _chunk_rows(c, b)
        fw = chunk_forward(h[s], r[s], tgt[s], W, gf, head, eps)
        _, bw = chunk_grad(fw, W, gf, head)
        return chunk_hvp(fw, bw, W, gf, head, eps, v)

    grad, L, _ = meta_grad(N, W0, eta, loss_grad, hvp)
    return grad, L, rows_loss


def adapted_loss_top_mlp(h, r, tgt, W0, gf, head, eta, eps, b):
    """L(W^(0)) alone (the inner loop of eq. (5), no meta-gradient)."""
    h, r, gf, head = (np.asarray(t, dtype=F) for t in (h, r, gf, head))
    tgt = np.asarray(tgt, dtype=np.int64)
    N = len(tgt) // b

    def loss_grad(c, W):
        s = _chunk_rows(c, b)
        fw = chunk_forward(h[s], r[s], tgt[s], W, gf, head, eps)
        g, _ = chunk_grad(fw, W, gf, head)
        return fw["A"], g

    _, losses = inner_loop(N, W0, eta, loss_grad)
    return float(np.mean(losses))
