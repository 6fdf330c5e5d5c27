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

``meta_grad_model`` takes eq. (7) over the whole model with fast MLPs in
every top block (n_u >= 1), where a chunk's loss reaches a lower fast MLP
through the upper blocks' attention: its Hessian-vector products carry the
tangent of the attention forward and backward too (see the section comment
further down for what is held fixed).

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


# ----------------------------------------------------------------------------
# the whole model: fast MLPs in every top block (n_u >= 1)
#
# With more than one fast block, a chunk's loss reaches a lower fast MLP
# through the upper blocks' attention, so H_c v needs the tangent of the
# attention forward and backward.  Eq. (7) is taken as written: A_c is the
# chunk loss as a function of W with the chunk's cached keys and values held
# (they were computed under earlier weights; reading 3 of ttt_oracle), the
# same A_c whose gradient the inner loop steps along.  With n_u = 1 this is
# the exact gradient of L (the function above); with n_u > 1 the pages'
# "main dependency" leaves out the path through the cached keys, and so does
# this.


def _norm_t(x, xt, g, eps):
    """Tangent of rmsnorm (last axis) along xt: (yt, rt)."""
    r = 1.0 / np.sqrt(np.mean(x * x, axis=-1, keepdims=True) + eps)
    rt = -r ** 3 * np.mean(x * xt, axis=-1, keepdims=True)
    return g * (xt * r + x * rt), rt


def _norm_bwd_t(x, xt, r, rt, g, dy, dyt):
    """Tangent of rmsnorm_bwd: dx = r u - r^3 x mean(x u), u = g dy."""
    u, ut = g * dy, g * dyt
    m = np.mean(x * u, axis=-1, keepdims=True)
    mt = np.mean(xt * u + x * ut, axis=-1, keepdims=True)
    return rt * u + r * ut - 3.0 * r * r * rt * x * m - r ** 3 * xt * m - r ** 3 * x * mt


def _swiglu_t(h, ht, w, v, G, U):
    """Forward tangent of swiglu along the input (ht) and the weights (v; None = fixed)."""
    wg, wu, wd = w
    sl, d1, _ = _silu_derivs(G)
    Gt = ht @ wg.T + (h @ v[0].T if v else 0.0)
    Ut = ht @ wu.T + (h @ v[1].T if v else 0.0)
    at = d1 * Gt * U + sl * Ut
    a = sl * U
    yt = at @ wd.T + (a @ v[2].T if v else 0.0)
    return Gt, Ut, at, yt


def _swiglu_bwd_t(dy, dyt, h, ht, G, U, Gt, Ut, at, w, v):
    """Primal and tangent of swiglu_bwd: (dh, dht, (grads), (grad tangents))."""
    wg, wu, wd = w
    sl, d1, d2 = _silu_derivs(G)
    a = sl * U
    da = dy @ wd
    dat = dyt @ wd + (dy @ v[2] if v else 0.0)
    dG = da * U * d1
    dU = da * sl
    dGt = dat * U * d1 + da * Ut * d1 + da * U * d2 * Gt
    dUt = dat * sl + da * d1 * Gt
    grads = (dG.T @ h, dU.T @ h, dy.T @ a)
    grads_t = (dGt.T @ h + dG.T @ ht, dUt.T @ h + dU.T @ ht, dyt.T @ a + dy.T @ at)
    dh = dG @ wg + dU @ wu
    dht = dGt @ wg + dUt @ wu + ((dG @ v[0] + dU @ v[1]) if v else 0.0)
    return dh, dht, grads, grads_t


def swa_tangent(q, K, V, P, qt, Kt, Vt):
    """Tangent of swa (ttt_oracle.swa, eq. (1) band) along (qt, Kt, Vt):
    St = scale (qt K^T + q Kt^T), Pt = P (St - rowsum(P St)), ot = Pt V + P Vt.
    Masked entries have P = 0, so they carry no tangent.  Returns (Pt, ot)."""
    scale = 1.0 / np.sqrt(q.shape[-1])
    St = (np.einsum("nhe,mhe->hnm", qt, K) + np.einsum("nhe,mhe->hnm", q, Kt)) * scale
    Pt = P * (St - np.sum(P * St, axis=-1, keepdims=True))
    ot = np.einsum("hnm,mhe->nhe", Pt, V) + np.einsum("hnm,mhe->nhe", P, Vt)
    return Pt, ot


def swa_bwd_tangent(do, dot, q, K, V, P, qt, Kt, Vt, Pt):
    """Tangent of swa_bwd (dq, dK, dV given dO) along the forward tangents
    (qt, Kt, Vt, Pt) and dot, the tangent of dO."""
    scale = 1.0 / np.sqrt(q.shape[-1])
    dP = np.einsum("nhe,mhe->hnm", do, V)
    dPt = np.einsum("nhe,mhe->hnm", dot, V) + np.einsum("nhe,mhe->hnm", do, Vt)
    dl = np.sum(dP * P, axis=-1, keepdims=True)
    dlt = np.sum(dPt * P + dP * Pt, axis=-1, keepdims=True)
    dS = P * (dP - dl)
    dSt = Pt * (dP - dl) + P * (dPt - dlt)
    dqt = (np.einsum("hnm,mhe->nhe", dSt, K) + np.einsum("hnm,mhe->nhe", dS, Kt)) * scale
    dKt = (np.einsum("hnm,nhe->mhe", dSt, q) + np.einsum("hnm,nhe->mhe", dS, qt)) * scale
    dVt = np.einsum("hnm,nhe->mhe", Pt, do) + np.einsum("hnm,nhe->mhe", P, dot)
    return dqt, dKt, dVt


def model_chunk_grad_hvp(model, W, fwd, weights, V):
    """(grad, H V) of A = sum_p weights[p] loss_p of one forwarded chunk
    (ttt_oracle.forward_chunk output) at fast weights W, cached keys held;
    V is a direction shaped like W.  The primal steps repeat
    ttt_oracle.backward_chunk; every step also carries its tangent."""
    from .ttt_oracle import rope, rope_bwd, swa_bwd
    cfg = model.cfg
    n, d, H, hd, eps = fwd["n"], cfg.d_model, cfg.n_heads, cfg.head_dim, cfg.norm_eps
    cos, sin = fwd["cos"], fwd["sin"]
    off = fwd["p0"] - fwd["kstart"]
    top = sorted(W)
    names = ("w_gate", "w_up", "w_down")
    # ---- forward tangent, lowest fast block upwards (its input does not depend on W)
    xt = np.zeros((n, d))
    T_ = {}
    for l in top:
        s = fwd["saved"][l]
        pre = f"layers.{l}."
        t = dict(x_in=xt)
        t["h"], t["r1"] = _norm_t(s["x_in"], xt, model[pre + "attn_norm"], eps)
        t["q"] = (t["h"] @ model[pre + "wq"].T).reshape(n, H, hd)
        t["kk"] = (t["h"] @ model[pre + "wk"].T).reshape(n, H, hd)
        t["v"] = (t["h"] @ model[pre + "wv"].T).reshape(n, H, hd)
        qnt, t["rq"] = _norm_t(s["q"], t["q"], model[pre + "q_norm"], eps)
        knt, t["rk"] = _norm_t(s["kk"], t["kk"], model[pre + "k_norm"], eps)
        t["qr"] = rope(qnt, cos, sin)
        Kwt = np.zeros_like(s["Kw"])
        Vwt = np.zeros_like(s["Vw"])
        Kwt[off:off + n] = rope(knt, cos, sin)
        Vwt[off:off + n] = t["v"]
        t["Kw"], t["Vw"] = Kwt, Vwt
        t["P"], ot = swa_tangent(s["qr"], s["Kw"], s["Vw"], s["P"], t["qr"], Kwt, Vwt)
        t["x_mid"] = xt + ot.reshape(n, d) @ model[pre + "wo"].T
        t["h2"], t["r2"] = _norm_t(s["x_mid"], t["x_mid"], model[pre + "mlp_norm"], eps)
        ws = (model[pre + "w_gate"], model[pre + "w_up"], model[pre + "w_down"])
        wf = tuple(W[l][nm] for nm in names)
        vf = tuple(V[l][nm] for nm in names)
        t["ms"] = _swiglu_t(s["h2"], t["h2"], ws, None, s["ms"][0], s["ms"][1])
        t["mf"] = _swiglu_t(s["h2"], t["h2"], wf, vf, s["mf"][0], s["mf"][1])
        xt = t["x_mid"] + t["ms"][3] + t["mf"][3]
        T_[l] = t
    hft, rft = _norm_t(fwd["x"], xt, model["final_norm"], eps)
    zt = hft @ model["lm_head"].T
    # ---- backward and its tangent
    valid, tgt = fwd["valid"], fwd["tgt"]
    rows = np.nonzero(valid)[0]
    Pz = fwd["probs"]
    dz = np.zeros((n, cfg.vocab))
    dzt = np.zeros((n, cfg.vocab))
    wv = weights[valid][:, None]
    dzv = Pz.copy()
    dzv[np.arange(len(rows)), tgt[valid]] -= 1.0
    dz[valid] = dzv * wv
    ztv = zt[valid]
    dzt[valid] = wv * Pz * (ztv - np.sum(Pz * ztv, axis=-1, keepdims=True))
    head = model["lm_head"]
    dhf, dhft = dz @ head, dzt @ head
    dx = rmsnorm_bwd(fwd["x"], fwd["rf"], model["final_norm"], dhf)
    dxt = _norm_bwd_t(fwd["x"], xt, fwd["rf"], rft, model["final_norm"], dhf, dhft)
    G, HV = {}, {}
    lowest = top[0]
    for l in reversed(top):
        s, t = fwd["saved"][l], T_[l]
        pre = f"layers.{l}."
        wf = tuple(W[l][nm] for nm in names)
        vf = tuple(V[l][nm] for nm in names)
        Gf, Uf, _ = s["mf"]
        Gft, Uft, aft, _ = t["mf"]
        dh2_f, dh2_ft, gr, grt = _swiglu_bwd_t(dx, dxt, s["h2"], t["h2"], Gf, Uf, Gft, Uft, aft, wf, vf)
        G[l] = dict(zip(names, gr))
        HV[l] = dict(zip(names, grt))
        if l == lowest:
            break  # nothing below the lowest fast block depends on W
        ws = (model[pre + "w_gate"], model[pre + "w_up"], model[pre + "w_down"])
        Gs, Us, _ = s["ms"]
        Gst, Ust, ast, _ = t["ms"]
        dh2_s, dh2_st, _, _ = _swiglu_bwd_t(dx, dxt, s["h2"], t["h2"], Gs, Us, Gst, Ust, ast, ws, None)
        g_m = model[pre + "mlp_norm"]
        dx_mid = dx + rmsnorm_bwd(s["x_mid"], s["r2"], g_m, dh2_s + dh2_f)
        dx_midt = dxt + _norm_bwd_t(s["x_mid"], t["x_mid"], s["r2"], t["r2"], g_m, dh2_s + dh2_f, dh2_st + dh2_ft)
        wo = model[pre + "wo"]
        do = (dx_mid @ wo).reshape(n, H, hd)
        dot = (dx_midt @ wo).reshape(n, H, hd)
        # attention backward (primal as ttt_oracle.swa_bwd) and its tangent
        P, Pt = s["P"], t["P"]
        dq_r, dK, dV = swa_bwd(do, s["qr"], s["Kw"], s["Vw"], P, hd)
        dq_rt, dKt, dVt = swa_bwd_tangent(do, dot, s["qr"], s["Kw"], s["Vw"], P, t["qr"], t["Kw"], t["Vw"], Pt)
        dk_r, dv = dK[off:off + n], dV[off:off + n]
        dk_rt, dvt = dKt[off:off + n], dVt[off:off + n]
        dqn, dqnt = rope_bwd(dq_r, cos, sin), rope_bwd(dq_rt, cos, sin)
        dkn, dknt = rope_bwd(dk_r, cos, sin), rope_bwd(dk_rt, cos, sin)
        gq, gk = model[pre + "q_norm"], model[pre + "k_norm"]
        dq = rmsnorm_bwd(s["q"], s["rq"], gq, dqn)
        dqt = _norm_bwd_t(s["q"], t["q"], s["rq"], t["rq"], gq, dqn, dqnt)
        dk = rmsnorm_bwd(s["kk"], s["rk"], gk, dkn)
        dkt = _norm_bwd_t(s["kk"], t["kk"], s["rk"], t["rk"], gk, dkn, dknt)
        wq, wk, wvv = model[pre + "wq"], model[pre + "wk"], model[pre + "wv"]
        dh = dq.reshape(n, d) @ wq + dk.reshape(n, d) @ wk + dv.reshape(n, d) @ wvv
        dht = dqt.reshape(n, d) @ wq + dkt.reshape(n, d) @ wk + dvt.reshape(n, d) @ wvv
        g_a = model[pre + "attn_norm"]
        dx = dx_mid + rmsnorm_bwd(s["x_in"], s["r1"], g_a, dh)
        dxt = dx_midt + _norm_bwd_t(s["x_in"], t["x_in"], s["r1"], t["r1"], g_a, dh, dht)
    return G, HV


def _flat(W):
    return tuple(W[l][nm] for l in sorted(W) for nm in ("w_gate", "w_up", "w_down"))


def _unflat(t, like):
    out, i = {}, 0
    for l in sorted(like):
        out[l] = {}
        for nm in ("w_gate", "w_up", "w_down"):
            out[l][nm] = t[i]
            i += 1
    return out


def _chunk_targets(toks, p0, n):
    tgt = np.full(n, -1, dtype=np.int64)
    nt = min(n, len(toks) - 1 - p0)
    if nt > 0:
        tgt[:nt] = toks[p0 + 1:p0 + 1 + nt]
    return tgt


def meta_grad_model(model, toks, eta=None):
    """eq. (7) for every fast MLP of the model over the sequence's full
    chunks: (grad as {block: {name: array}}, L, per-chunk A_c).  Each chunk's
    loss is taken with its cached keys and values as the inner loop computed
    them (see the section comment)."""
    from .ttt_oracle import State, forward_chunk, init_fast
    cfg = model.cfg
    eta = cfg.eta if eta is None else eta
    toks = np.asarray(toks, dtype=np.int64)
    b = cfg.b
    N = len(toks) // b
    state = State(cfg, len(toks))
    like = init_fast(model)

    def fwd_of(c, Wt):
        p0 = c * b
        tgt = _chunk_targets(toks, p0, b)
        loss, fwd = forward_chunk(model, _unflat(Wt, like), state, toks[p0:p0 + b], p0, tgt)
        nc = int((tgt >= 0).sum())
        wts = np.where(tgt >= 0, 1.0 / nc, 0.0) if nc else np.zeros(b)
        return loss, fwd, wts, nc

    def loss_grad(c, Wt):
        loss, fwd, wts, nc = fwd_of(c, Wt)
        if nc == 0:
            return 0.0, tuple(np.zeros_like(w) for w in Wt)
        G, _ = model_chunk_grad_hvp(model, _unflat(Wt, like), fwd, wts, _unflat(tuple(np.zeros_like(w) for w in Wt), like))
        return float(np.nanmean(loss)), _flat(G)

    def hvp(c, Wt, v):
        loss, fwd, wts, nc = fwd_of(c, Wt)
        if nc == 0:
            return tuple(np.zeros_like(w) for w in Wt)
        _, HV = model_chunk_grad_hvp(model, _unflat(Wt, like), fwd, wts, _unflat(v, like))
        return _flat(HV)

    g, L, losses = meta_grad(N, _flat(like), eta, loss_grad, hvp)
    return _unflat(g, like), L, losses


def frozen_adapted_loss(model, toks, W0, cache, eta=None):
    """L of the inner loop started at W0 (dict like init_fast), every chunk's
    keys and values of earlier positions taken from ``cache`` (a State of an
    unperturbed run) instead of this run's: the function whose gradient at
    the unperturbed W0 is eq. (7) as taken above."""
    from .ttt_oracle import State, backward_chunk, forward_chunk
    cfg = model.cfg
    eta = cfg.eta if eta is None else eta
    toks = np.asarray(toks, dtype=np.int64)
    b = cfg.b
    N = len(toks) // b
    W = {l: {nm: np.array(a, dtype=F) for nm, a in W0[l].items()} for l in W0}
    state = State(cfg, len(toks))
    means = []
    for c in range(N):
        p0 = c * b
        for l in range(cfg.n_layers):
            state.K[l][:p0] = cache.K[l][:p0]
            state.V[l][:p0] = cache.V[l][:p0]
        tgt = _chunk_targets(toks, p0, b)
        loss, fwd = forward_chunk(model, W, state, toks[p0:p0 + b], p0, tgt)
        nc = int((tgt >= 0).sum())
        means.append(float(np.nanmean(loss)) if nc else 0.0)
        if nc:
            G = backward_chunk(model, W, fwd, np.where(tgt >= 0, 1.0 / nc, 0.0))
            for l in G:
                for nm in G[l]:
                    W[l][nm] = W[l][nm] - eta * G[l][nm]
    return float(np.mean(means))
