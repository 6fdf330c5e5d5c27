"""CPU oracle of the TTT-E2E prefill loop — TEST INFRASTRUCTURE ONLY.

Only ``tests/``, ``__graft_entry__.smoke()`` and the ``cpu_baseline`` /
``--impl reference`` legs of ``bench.py`` may import this module.  The CUDA
library never calls it, and it shares no code with the CUDA library: only
the seeded input generators in ``synth/`` feed both.

It is a plain, slow, fp64 numpy restatement of the method, taken step by step
in the order of the pages (End-to-End Test-Time Training for Long Context;
reading notes by Zhongzhu Zhou, "算法 1：因果预填充与内层适应" and eq. (9)):

  1. copy the fast weights W <- W_init, empty attention state;
  2. for each chunk of b tokens, in order:
       forward every position with the current W (the Transformer with
       sliding-window attention, eq. (1)); record the next-token loss of
       every position *before* any update (reading notes §7, 算法 1);
       A_c = mean loss over the chunk's targets, eq. (9);
       G = dA_c/dW by an explicit, hand-derived backward;
       W <- W - eta * G (plain SGD, eq. (9));
       keep the keys/values the window still needs (算法 1);
  3. return the per-token losses and the adapted W.

Only the MLPs of the last n_u blocks carry fast weights (the reading notes,
§6, restrict the inner-loop update to the MLPs of the final quarter of the
blocks); each such block keeps a static MLP beside the fast one and sums
their outputs (reading notes §6, second paragraph; reportify.cn, the section
on the dual-MLP structure).  Everything else is frozen in the inner loop.

Readings where the pages are silent:
  * position p (0-based) predicts tokens[p+1]; the last position has no
    target (loss NaN); A_c divides by the number n_c of targets in the chunk;
  * keys of earlier chunks are the values cached when those positions were
    processed; they are constants of the current chunk's gradient;
  * a trailing partial chunk is scored but does not update W (its update
    would wait for more tokens, as in generation, 算法 3);
  * RMSNorm y = x / sqrt(mean(x^2) + eps) * g, eps = 1e-5; QK-norm is a
    per-head RMSNorm over head_dim applied before RoPE; RoPE pairs element i
    with i + hd/2 at absolute position p, theta = 10000; attention scale is
    1/sqrt(hd); SwiGLU(h) = (silu(h Wg^T) * (h Wu^T)) Wd^T;
  * window k: query p sees keys j with p-k+1 <= j <= p (min(p+1, k) keys,
    eq. (1) counted 1-based).

All arithmetic is float64.  Weights arrive as float32 arrays (for bf16
configs they already hold the bf16-rounded values both sides use).
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field

import numpy as np

F = np.float64


# ----------------------------------------------------------------------------
# building blocks


def rmsnorm(x, g, eps):
    """y = x * r * g with r = 1/sqrt(mean(x^2) + eps) over the last axis."""
    r = 1.0 / np.sqrt(np.mean(x * x, axis=-1, keepdims=True) + eps)
    return x * r * g, r


def rmsnorm_bwd(x, r, g, dy):
    """Gradient of rmsnorm w.r.t. x:  r * (u - xh * mean(xh * u)),
    u = dy * g, xh = x * r  (differentiate x_i * r(x) * g_i; dr/dx_j = -r^3 x_j / n)."""
    xh = x * r
    u = dy * g
    return r * (u - xh * np.mean(xh * u, axis=-1, keepdims=True))


def rope_tables(pos, hd, theta):
    """cos, sin of angle p * theta^(-2i/hd), i < hd/2, for absolute positions p."""
    i = np.arange(hd // 2, dtype=F)
    inv = theta ** (-2.0 * i / hd)
    ang = np.asarray(pos, dtype=F)[:, None] * inv[None, :]
    return np.cos(ang), np.sin(ang)


def rope(x, cos, sin):
    """Rotate pairs (i, i + hd/2) of x [n, H, hd] by the position angle."""
    h2 = x.shape[-1] // 2
    c, s = cos[:, None, :], sin[:, None, :]
    x1, x2 = x[..., :h2], x[..., h2:]
    return np.concatenate([x1 * c - x2 * s, x2 * c + x1 * s], axis=-1)


def rope_bwd(dy, cos, sin):
    """Transpose of the rotation (rotation by minus the angle)."""
    h2 = dy.shape[-1] // 2
    c, s = cos[:, None, :], sin[:, None, :]
    d1, d2 = dy[..., :h2], dy[..., h2:]
    return np.concatenate([d1 * c + d2 * s, d2 * c - d1 * s], axis=-1)


def sigmoid(x):
    return 0.5 * (1.0 + np.tanh(0.5 * x))


def swiglu(h, wg, wu, wd):
    """y = (silu(h wg^T) * (h wu^T)) wd^T; returns y and (g, u, a)."""
    g = h @ wg.T
    u = h @ wu.T
    a = g * sigmoid(g) * u
    return a @ wd.T, (g, u, a)


def swiglu_bwd(dy, h, g, u, a, wg, wu, wd, need_dh=True):
    """Backward of swiglu: returns dh (or None) and (dwg, dwu, dwd)."""
    sg = sigmoid(g)
    da = dy @ wd                       # [n, f]
    dg = da * u * sg * (1.0 + g * (1.0 - sg))   # d silu(g)/dg = s(g)(1 + g(1 - s(g)))
    du = da * g * sg
    dwd = dy.T @ a                     # [d, f]
    dwg = dg.T @ h                     # [f, d]
    dwu = du.T @ h
    dh = dg @ wg + du @ wu if need_dh else None
    return dh, (dwg, dwu, dwd)


def window_mask(qpos, kpos, k):
    """Boolean [nq, nk]: key j visible to query p iff p-k+1 <= j <= p."""
    qp = np.asarray(qpos)[:, None]
    kp = np.asarray(kpos)[None, :]
    return (kp <= qp) & (kp > qp - k)


def swa(q, K, V, qpos, kpos, k):
    """Sliding-window causal attention, eq. (1).
    q [n, H, hd]; K, V [m, H, hd] at absolute positions kpos; returns o, P."""
    hd = q.shape[-1]
    s = np.einsum("nhe,mhe->hnm", q, K) / math.sqrt(hd)
    mask = window_mask(qpos, kpos, k)[None]
    s = np.where(mask, s, -np.inf)
    s = s - s.max(axis=-1, keepdims=True)
    P = np.exp(s)
    P = P / P.sum(axis=-1, keepdims=True)
    o = np.einsum("hnm,mhe->nhe", P, V)
    return o, P


def swa_bwd(do, q, K, V, P, hd):
    """Backward of swa w.r.t. q, K, V (full key set given)."""
    scale = 1.0 / math.sqrt(hd)
    dP = np.einsum("nhe,mhe->hnm", do, V)
    dV = np.einsum("hnm,nhe->mhe", P, do)
    dS = P * (dP - np.sum(dP * P, axis=-1, keepdims=True))
    dq = np.einsum("hnm,mhe->nhe", dS, K) * scale
    dK = np.einsum("hnm,nhe->mhe", dS, q) * scale
    return dq, dK, dV


def log_softmax_ce(z, targets):
    """Per-row natural-log cross-entropy -log softmax(z)[t]; also softmax(z)."""
    m = z.max(axis=-1, keepdims=True)
    e = np.exp(z - m)
    ssum = e.sum(axis=-1, keepdims=True)
    lse = (m + np.log(ssum))[:, 0]
    loss = lse - z[np.arange(z.shape[0]), targets]
    return loss, e / ssum, lse


# ----------------------------------------------------------------------------
# model


@dataclass
class Model:
    """Static weights phi (float64 views built lazily) plus config."""

    cfg: object
    w: dict            # name -> float32 array (synth.Weights.arrays)
    _cache: dict = field(default_factory=dict)
    cache_budget: int = 1 << 28   # float64 elements kept widened between uses

    def __getitem__(self, name):
        a = self._cache.get(name)
        if a is None:
            a = np.asarray(self.w[name], dtype=F)
            if a.size <= self.cache_budget:
                self._cache[name] = a
                self.cache_budget -= a.size
        return a

    def rows(self, name, idx):
        """float64 copy of selected rows (embedding lookup)."""
        return np.asarray(self.w[name][idx], dtype=F)

    @property
    def top(self):
        L, nu = self.cfg.n_layers, self.cfg.n_updated
        return list(range(L - nu, L))


def init_fast(model):
    """W <- W_init (start of 算法 1): float64 copies of every fast tensor."""
    return {l: {"w_gate": np.array(model.w[f"fast.{l}.w_gate"], dtype=F),
                "w_up": np.array(model.w[f"fast.{l}.w_up"], dtype=F),
                "w_down": np.array(model.w[f"fast.{l}.w_down"], dtype=F)} for l in model.top}


class State:
    """Attention state carried across chunks: the rotated keys and the values
    of every processed position, per block.  The window mask restricts what
    a query may read, so keeping more than the window changes nothing."""

    def __init__(self, cfg, T):
        H, hd = cfg.n_heads, cfg.head_dim
        self.K = [np.zeros((T, H, hd)) for _ in range(cfg.n_layers)]
        self.V = [np.zeros((T, H, hd)) for _ in range(cfg.n_layers)]
        self.pairs = 0  # query-key pairs admitted by the window (eq. (1) check)


def forward_chunk(model, W, state, toks, p0, tgt, fast_on=True, count_pairs=False):
    """Forward positions p0 .. p0+n-1 through all blocks with fast weights W.
    Writes their keys/values into ``state``.  Returns per-position loss
    (NaN where tgt < 0) and the saved activations of the top blocks."""
    cfg = model.cfg
    n = len(toks)
    L, d, H, hd, eps = cfg.n_layers, cfg.d_model, cfg.n_heads, cfg.head_dim, cfg.norm_eps
    k = cfg.k
    pos = np.arange(p0, p0 + n)
    cos, sin = rope_tables(pos, hd, cfg.rope_theta)
    kstart = max(0, p0 - k + 1)
    kpos = np.arange(kstart, p0 + n)
    x = model.rows("embed", toks)
    saved = {}
    for l in range(L):
        pre = f"layers.{l}."
        x_in = x
        h, r1 = rmsnorm(x, model[pre + "attn_norm"], eps)
        q = (h @ model[pre + "wq"].T).reshape(n, H, hd)
        kk = (h @ model[pre + "wk"].T).reshape(n, H, hd)
        v = (h @ model[pre + "wv"].T).reshape(n, H, hd)
        qn, rq = rmsnorm(q, model[pre + "q_norm"], eps)
        kn, rk = rmsnorm(kk, model[pre + "k_norm"], eps)
        qr, kr = rope(qn, cos, sin), rope(kn, cos, sin)
        state.K[l][p0:p0 + n] = kr
        state.V[l][p0:p0 + n] = v
        Kw, Vw = state.K[l][kstart:p0 + n], state.V[l][kstart:p0 + n]
        o, P = swa(qr, Kw, Vw, pos, kpos, k)
        if count_pairs and l == 0:
            state.pairs += int(window_mask(pos, kpos, k).sum())
        x = x + o.reshape(n, d) @ model[pre + "wo"].T
        x_mid = x
        h2, r2 = rmsnorm(x, model[pre + "mlp_norm"], eps)
        y, ms = swiglu(h2, model[pre + "w_gate"], model[pre + "w_up"], model[pre + "w_down"])
        mf = None
        if fast_on and l in W:
            yf, mf = swiglu(h2, W[l]["w_gate"], W[l]["w_up"], W[l]["w_down"])
            y = y + yf
        x = x_mid + y
        if l in W:
            saved[l] = dict(x_in=x_in, r1=r1, h=h, q=q, kk=kk, rq=rq, rk=rk, qr=qr, v=v, o=o, P=P,
                            Kw=Kw, Vw=Vw, x_mid=x_mid, r2=r2, h2=h2, ms=ms, mf=mf)
    hf, rf = rmsnorm(x, model["final_norm"], eps)
    z = hf @ model["lm_head"].T
    valid = tgt >= 0
    loss = np.full(n, np.nan)
    loss_v, probs, _ = log_softmax_ce(z[valid], tgt[valid])
    loss[valid] = loss_v
    return loss, dict(saved=saved, x=x, rf=rf, hf=hf, probs=probs, valid=valid, tgt=tgt, z_last=z[n - 1].copy(),
                      cos=cos, sin=sin, n=n, p0=p0, kstart=kstart)


def backward_chunk(model, W, fwd, weights):
    """G = dA/dW for A = sum_p weights[p] * loss_p over valid positions p.
    Explicit backward through the top blocks only: below block L-n_u nothing
    depends on W (reading notes §6; the hyper.ai summary: gradients reach
    only the updated layers)."""
    cfg = model.cfg
    n, d, H, hd, eps = fwd["n"], cfg.d_model, cfg.n_heads, cfg.head_dim, cfg.norm_eps
    valid, tgt = fwd["valid"], fwd["tgt"]
    # dA/dz = w_p (softmax - onehot) on valid rows
    dz = np.zeros((n, cfg.vocab))
    dzv = fwd["probs"].copy()
    dzv[np.arange(dzv.shape[0]), tgt[valid]] -= 1.0
    dz[valid] = dzv * weights[valid][:, None]
    dhf = dz @ model["lm_head"]
    dx = rmsnorm_bwd(fwd["x"], fwd["rf"], model["final_norm"], dhf)
    G = {}
    lowest = min(W)
    for l in sorted(W, reverse=True):
        s = fwd["saved"][l]
        pre = f"layers.{l}."
        # MLP sub-block: x_out = x_mid + MLP_s(h2) + MLP_f(h2)
        g_f, u_f, a_f = s["mf"]
        need = l > lowest
        dh2_f, (dwg, dwu, dwd) = swiglu_bwd(dx, s["h2"], g_f, u_f, a_f,
                                            W[l]["w_gate"], W[l]["w_up"], W[l]["w_down"], need)
        G[l] = {"w_gate": dwg, "w_up": dwu, "w_down": dwd}
        if not need:
            break  # nothing below the lowest fast block depends on W
        g_s, u_s, a_s = s["ms"]
        dh2_s, _ = swiglu_bwd(dx, s["h2"], g_s, u_s, a_s, model[pre + "w_gate"], model[pre + "w_up"],
                              model[pre + "w_down"], True)
        dx_mid = dx + rmsnorm_bwd(s["x_mid"], s["r2"], model[pre + "mlp_norm"], dh2_s + dh2_f)
        # attention sub-block: x_mid = x_in + o Wo^T
        do = (dx_mid @ model[pre + "wo"]).reshape(n, H, hd)
        # keys of earlier chunks are constants: only this chunk's keys get gradients
        dq_r, dK, dV = swa_bwd(do, s["qr"], s["Kw"], s["Vw"], s["P"], hd)
        off = fwd["p0"] - fwd["kstart"]
        dk_r, dv = dK[off:off + n], dV[off:off + n]
        dqn = rope_bwd(dq_r, fwd["cos"], fwd["sin"])
        dkn = rope_bwd(dk_r, fwd["cos"], fwd["sin"])
        dq = rmsnorm_bwd(s["q"], s["rq"], model[pre + "q_norm"], dqn)
        dk = rmsnorm_bwd(s["kk"], s["rk"], model[pre + "k_norm"], dkn)
        dh = (dq.reshape(n, d) @ model[pre + "wq"] + dk.reshape(n, d) @ model[pre + "wk"]
              + dv.reshape(n, d) @ model[pre + "wv"])
        dx = dx_mid + rmsnorm_bwd(s["x_in"], s["r1"], model[pre + "attn_norm"], dh)
    return G


@dataclass
class Result:
    losses: np.ndarray           # [T] float64, NaN at T-1
    W: dict                      # final fast weights (float64)
    chunk_mean: list             # A_c per chunk (mean over its targets)
    pairs: int = 0               # window pairs of block 0 (eq. (1))
    grads: list = None           # per updated chunk G (when keep_grads)
    state: object = None         # attention state after the last position (when keep_state)
    z_last: np.ndarray = None    # logits of position T-1, scored before its chunk's update


def prefill(model, toks, eta=None, b=None, k=None, keep_grads=False, count_pairs=False,
            n_chunks=None, keep_state=False, capacity=None):
    """The TTT prefill loop (算法 1).  ``toks`` int array of length T.
    Overrides of eta/b/k default to the config's.  ``n_chunks`` stops early
    (prefix runs).  Returns Result."""
    cfg = model.cfg
    if k is not None or b is not None:
        cfg = cfg.with_(k=cfg.k if k is None else k, b=cfg.b if b is None else b)
        model = Model(cfg, model.w, model._cache, model.cache_budget)
    eta = cfg.eta if eta is None else eta
    T, b = len(toks), cfg.b
    toks = np.asarray(toks, dtype=np.int64)
    W = init_fast(model)
    state = State(cfg, max(T, capacity or 0))  # room for positions generated later (decode)
    losses = np.full(T, np.nan)
    means, grads = [], []
    z_last = None
    nch = -(-T // b)
    if n_chunks is not None:
        nch = min(nch, n_chunks)
    for c in range(nch):
        p0 = c * b
        n = min(b, T - p0)
        tgt = np.full(n, -1, dtype=np.int64)
        nt = min(n, T - 1 - p0)
        if nt > 0:
            tgt[:nt] = toks[p0 + 1:p0 + 1 + nt]
        loss, fwd = forward_chunk(model, W, state, toks[p0:p0 + n], p0, tgt, count_pairs=count_pairs)
        losses[p0:p0 + n] = loss          # recorded before the update
        z_last = fwd["z_last"]
        n_c = int((tgt >= 0).sum())
        means.append(float(np.nanmean(loss)) if n_c else float("nan"))
        if n == b and n_c > 0 and W:
            wts = np.where(tgt >= 0, 1.0 / n_c, 0.0)
            G = backward_chunk(model, W, fwd, wts)
            for l in G:
                for name in G[l]:
                    W[l][name] = W[l][name] - eta * G[l][name]   # eq. (9)
            if keep_grads:
                grads.append(G)
    return Result(losses, W, means, state.pairs, grads if keep_grads else None,
                  state if keep_state else None, z_last)


@dataclass
class DecodeResult:
    tokens: np.ndarray           # [n_gen] generated token ids
    losses: np.ndarray           # [n_gen] loss of the position before each generated token, against it
    W: dict                      # fast weights after the last completed chunk
    updates: list                # positions p after whose forward a chunk [p+1-b, p] updated W
    prefill: Result              # the prefill of the prompt
    gaps: np.ndarray = None      # [n_gen] largest minus second-largest logit at each pick


def decode(model, prompt, n_gen, eta=None):
    """Greedy generation with periodic fast-weight updates (算法 3 of the
    reading notes: generate causally from the state the prefill left, collect
    the generated tokens until an inner chunk is full, take that chunk's
    next-token loss, update the fast weights, continue from the new state).

    Readings where the pages are silent:
      * greedy: the next token is the argmax of the logits of the position
        before it, ties to the lowest token id (np.argmax keeps the first);
      * chunks keep the prefill's grid of absolute positions [cb, (c+1)b): a
        trailing partial prompt chunk (scored but not applied by the
        prefill) is completed by the first generated tokens and then
        applied; the page names the half chunk as an open serving question;
      * a position is scored with the fast weights of its chunk, before that
        chunk's update: the token after position T-1 comes from the logits
        the prefill computed for T-1, and the token after the last position
        of a chunk from that position's pre-update logits;
      * the chunk's update is the prefill's: the mean loss over its b
        targets, the explicit backward, one SGD step (eq. (9))."""
    cfg = model.cfg
    b = cfg.b
    eta = cfg.eta if eta is None else eta
    prompt = np.asarray(prompt, dtype=np.int64)
    T = len(prompt)
    pre = prefill(model, prompt, eta=eta, keep_state=True, capacity=T + n_gen)
    W, state = pre.W, pre.state
    toks = [int(t) for t in prompt]
    z = pre.z_last  # logits of position T-1
    gen, losses, updates, gaps = [], [], [], []
    none = np.full(1, -1, dtype=np.int64)
    for p in range(T, T + n_gen):
        x = int(np.argmax(z))
        gaps.append(float(z[x] - np.max(np.delete(z, x))) if len(z) > 1 else float("inf"))
        m = z.max()
        losses.append(float(m + np.log(np.exp(z - m).sum()) - z[x]))
        gen.append(x)
        toks.append(x)
        # forward of position p with the current fast weights (keys/values cached in `state`)
        _, fwd = forward_chunk(model, W, state, np.asarray([x]), p, none)
        z = fwd["z_last"]
        if (p + 1) % b == 0:
            # chunk [c0, p] is complete: every target is known once position p's argmax is
            c0 = p + 1 - b
            tgt = np.asarray(toks[c0 + 1:p + 1] + [int(np.argmax(z))], dtype=np.int64)
            # its forward again, in one pass: the same W and cached keys give the same values
            _, cf = forward_chunk(model, W, state, np.asarray(toks[c0:p + 1]), c0, tgt)
            G = backward_chunk(model, W, cf, np.full(b, 1.0 / b))
            for l in G:
                for name in G[l]:
                    W[l][name] = W[l][name] - eta * G[l][name]   # eq. (9)
            updates.append(p)
    return DecodeResult(np.asarray(gen, dtype=np.int64), np.asarray(losses), W, updates, pre, np.asarray(gaps))


def static_losses(model, toks, k=None, fast=None):
    """Losses of the whole sequence in one forward pass with fixed fast
    weights (L_static of eq. (4)); W_init unless ``fast`` is given."""
    cfg = model.cfg if k is None else model.cfg.with_(k=k)
    m = Model(cfg, model.w, model._cache, model.cache_budget)
    T = len(toks)
    toks = np.asarray(toks, dtype=np.int64)
    W = init_fast(m) if fast is None else fast
    tgt = np.full(T, -1, dtype=np.int64)
    tgt[:T - 1] = toks[1:]
    loss, _ = forward_chunk(m, W, State(cfg, T), toks, 0, tgt)
    return loss


def window_pairs(T, k):
    """Number of (query, key) pairs admitted by the window, eq. (1):
    sum_{t=1}^{T} min(t, k)."""
    return sum(min(t, k) for t in range(1, T + 1))
