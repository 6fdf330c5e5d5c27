"""Pins of the meta-gradient oracle (oracle/meta_grad.py) to facts outside
itself (CPU only): central finite differences of the chunk loss, of its
gradient and of the adapted loss L(W^(0)); the symmetry of the Hessian; the
scalar quadratic of eq. (8) and a matrix quadratic in closed form; the
special cases eta = 0 (eq. (4), L_static) and one chunk; and the full model
oracle with only its last block updated (End-to-End Test-Time Training for
Long Context; reading notes by Zhongzhu Zhou, §4, eqs. (4)-(8))."""
import numpy as np
import pytest

import synth
from oracle import meta_grad as M
from oracle import ttt_oracle as O


def _case(seed=0, n=7, d=8, f=12, V=11, n_chunks=1, invalid=(2,)):
    rng = np.random.default_rng(seed)
    N = n_chunks * n
    h = rng.standard_normal((N, d))
    r = rng.standard_normal((N, d))
    tgt = rng.integers(0, V, N)
    for i in invalid:
        tgt[i] = -1
    W = (0.4 * rng.standard_normal((f, d)), 0.4 * rng.standard_normal((f, d)), 0.4 * rng.standard_normal((d, f)))
    gf = 1.0 + 0.3 * rng.standard_normal(d)
    head = 0.5 * rng.standard_normal((V, d))
    return h, r, tgt, W, gf, head


def _dot(a, b):
    return sum(float(np.sum(x * y)) for x, y in zip(a, b))


def _rand_dir(W, seed):
    rng = np.random.default_rng(seed)
    return tuple(rng.standard_normal(w.shape) for w in W)


EPS = 1e-5


def _fd(fun, W, v, e=1e-4):
    """Directional derivative of fun at W along v by the five-point central
    stencil (truncation error O(e^4))."""
    f = lambda t: fun(M._axpy(W, t, v))
    return (8.0 * (f(e) - f(-e)) - (f(2 * e) - f(-2 * e))) / (12.0 * e)


def _A(h, r, tgt, W, gf, head):
    return M.chunk_forward(h, r, tgt, W, gf, head, EPS)["A"]


def _g(h, r, tgt, W, gf, head):
    fw = M.chunk_forward(h, r, tgt, W, gf, head, EPS)
    return M.chunk_grad(fw, W, gf, head)[0]


def test_chunk_grad_matches_finite_differences():
    h, r, tgt, W, gf, head = _case()
    g = _g(h, r, tgt, W, gf, head)
    for s in range(3):
        v = _rand_dir(W, 10 + s)
        e = 1e-5
        fd = (_A(h, r, tgt, M._axpy(W, e, v), gf, head) - _A(h, r, tgt, M._axpy(W, -e, v), gf, head)) / (2 * e)
        assert abs(fd - _dot(g, v)) <= 1e-8 * max(1.0, abs(fd))


def test_hvp_matches_finite_differences_of_the_gradient():
    h, r, tgt, W, gf, head = _case(seed=1)
    fw = M.chunk_forward(h, r, tgt, W, gf, head, EPS)
    _, bw = M.chunk_grad(fw, W, gf, head)
    v = _rand_dir(W, 3)
    Hv = M.chunk_hvp(fw, bw, W, gf, head, EPS, v)
    e = 1e-5
    gp = _g(h, r, tgt, M._axpy(W, e, v), gf, head)
    gm = _g(h, r, tgt, M._axpy(W, -e, v), gf, head)
    for a, p, m in zip(Hv, gp, gm):
        fd = (p - m) / (2 * e)
        assert np.abs(a - fd).max() <= 1e-7 * np.abs(fd).max()


def test_hvp_is_symmetric():
    h, r, tgt, W, gf, head = _case(seed=2)
    fw = M.chunk_forward(h, r, tgt, W, gf, head, EPS)
    _, bw = M.chunk_grad(fw, W, gf, head)
    u, v = _rand_dir(W, 4), _rand_dir(W, 5)
    a = _dot(v, M.chunk_hvp(fw, bw, W, gf, head, EPS, u))
    b = _dot(u, M.chunk_hvp(fw, bw, W, gf, head, EPS, v))
    assert abs(a - b) <= 1e-12 * max(1.0, abs(a))


@pytest.mark.parametrize("eta", [0.3, 1.5])
def test_meta_grad_matches_finite_differences_of_the_adapted_loss(eta):
    n, N = 6, 4
    h, r, tgt, W, gf, head = _case(seed=6, n=n, n_chunks=N, invalid=(3, 23))
    grad, L, _ = M.meta_grad_top_mlp(h, r, tgt, W, gf, head, eta, EPS, n)
    assert abs(L - M.adapted_loss_top_mlp(h, r, tgt, W, gf, head, eta, EPS, n)) < 1e-14
    # the second-order path must matter for this case, or the check below would not see it
    first_order = tuple(sum(gi) / N for gi in zip(*[
        _g(h[c * n:(c + 1) * n], r[c * n:(c + 1) * n], tgt[c * n:(c + 1) * n], W, gf, head) for c in range(N)]))
    for s in range(3):
        v = _rand_dir(W, 20 + s)
        fd = _fd(lambda Wx: M.adapted_loss_top_mlp(h, r, tgt, Wx, gf, head, eta, EPS, n), W, v)
        assert abs(fd - _dot(grad, v)) <= 1e-7 * max(1.0, abs(fd))
        assert abs(fd - _dot(first_order, v)) > 1e-4 * max(1.0, abs(fd))


def test_scalar_quadratic_eq8_closed_form():
    """A_c(w) = a (w - w*)^2 / 2 for every chunk: e_c = (1 - eta a)^c e_0
    (eq. (8)), so dL/dw0 = (1/N) sum_c a (1 - eta a)^(2c) e_0."""
    a, ws, w0, N = 1.3, 1.0, 0.0, 6
    for eta in (0.2, 0.9, 1.6):
        lg = lambda c, W: (0.5 * a * float((W[0] - ws) ** 2), (a * (W[0] - ws),))
        hv = lambda c, W, v: (a * v[0],)
        grad, L, losses = M.meta_grad(N, (np.array(w0),), eta, lg, hv)
        e0 = w0 - ws
        want = sum(a * (1 - eta * a) ** (2 * c) * e0 for c in range(N)) / N
        assert abs(float(grad[0]) - want) <= 1e-14
        assert abs(L - sum(0.5 * a * ((1 - eta * a) ** c * e0) ** 2 for c in range(N)) / N) <= 1e-14


def test_matrix_quadratic_against_the_explicit_jacobian_product():
    """A_c(w) = (w - s_c)^T Q_c (w - s_c) / 2 with a different SPD Q_c per
    chunk: J_c = (I - eta Q_(c-1)) ... (I - eta Q_0) multiplied out in
    forward order, grad = (1/N) sum_c J_c^T Q_c (w_c - s_c)."""
    rng = np.random.default_rng(7)
    n, N, eta = 5, 5, 0.15
    Qs = []
    for _ in range(N):
        B = rng.standard_normal((n, n))
        Qs.append(B @ B.T / n + 0.1 * np.eye(n))
    S = [rng.standard_normal(n) for _ in range(N)]
    w0 = rng.standard_normal(n)
    lg = lambda c, W: (0.5 * float((W[0] - S[c]) @ Qs[c] @ (W[0] - S[c])), (Qs[c] @ (W[0] - S[c]),))
    hv = lambda c, W, v: (Qs[c] @ v[0],)
    grad, L, _ = M.meta_grad(N, (w0,), eta, lg, hv)
    J = np.eye(n)
    w = w0.copy()
    want = np.zeros(n)
    for c in range(N):
        want += J.T @ (Qs[c] @ (w - S[c])) / N
        w = w - eta * Qs[c] @ (w - S[c])
        J = (np.eye(n) - eta * Qs[c]) @ J
    assert np.abs(grad[0] - want).max() <= 1e-13


def test_eta_zero_is_the_static_gradient():
    """eta = 0: W never moves, L is L_static of eq. (4) by chunks and its
    gradient is the mean of the chunk gradients at W^(0)."""
    n, N = 5, 3
    h, r, tgt, W, gf, head = _case(seed=8, n=n, n_chunks=N, invalid=())
    grad, _, _ = M.meta_grad_top_mlp(h, r, tgt, W, gf, head, 0.0, EPS, n)
    gs = [_g(h[c * n:(c + 1) * n], r[c * n:(c + 1) * n], tgt[c * n:(c + 1) * n], W, gf, head) for c in range(N)]
    for i in range(3):
        assert np.abs(grad[i] - sum(g[i] for g in gs) / N).max() <= 1e-15


def test_one_chunk_is_its_own_gradient():
    h, r, tgt, W, gf, head = _case(seed=9)
    grad, L, rows = M.meta_grad_top_mlp(h, r, tgt, W, gf, head, 0.7, EPS, len(tgt))
    g = _g(h, r, tgt, W, gf, head)
    for a, b in zip(grad, g):
        assert np.array_equal(a, b)
    assert np.isnan(rows[2]) and np.isnan(rows).sum() == 1


def test_chunk_without_targets_contributes_nothing():
    n, N = 4, 3
    h, r, tgt, W, gf, head = _case(seed=10, n=n, n_chunks=N, invalid=(4, 5, 6, 7))
    assert M.chunk_forward(h[4:8], r[4:8], tgt[4:8], W, gf, head, EPS)["A"] == 0.0
    g = _g(h[4:8], r[4:8], tgt[4:8], W, gf, head)
    assert all(not np.any(x) for x in g)


MICRO = synth.ModelConfig("micro-meta", n_layers=2, d_model=16, n_heads=2, head_dim=8, d_ff=24, vocab=29,
                          n_updated=1, T=24, k=7, b=6, eta=0.8, dtype="f32", seed=0x3E7A)


def _inputs_of_the_last_block(model, toks, b):
    """h (MLP-norm output) and r (residual + static MLP) of the last block for
    every position, from the full oracle's forward; with n_u = 1 they do not
    depend on the fast weights."""
    cfg = model.cfg
    L = cfg.n_layers
    W = O.init_fast(model)
    state = O.State(cfg, len(toks))
    hs, rs = [], []
    for c in range(len(toks) // b):
        p0 = c * b
        tgt = np.full(b, -1, dtype=np.int64)
        nt = min(b, len(toks) - 1 - p0)
        tgt[:nt] = toks[p0 + 1:p0 + 1 + nt]
        _, fw = O.forward_chunk(model, W, state, toks[p0:p0 + b], p0, tgt)
        s = fw["saved"][L - 1]
        pre = f"layers.{L - 1}."
        y_s, _ = O.swiglu(s["h2"], model[pre + "w_gate"], model[pre + "w_up"], model[pre + "w_down"])
        hs.append(s["h2"])
        rs.append(s["x_mid"] + y_s)
    tg = np.full(len(toks), -1, dtype=np.int64)
    tg[:-1] = toks[1:]
    return np.concatenate(hs), np.concatenate(rs), tg


def test_matches_the_full_model_with_its_last_block_updated():
    """Directional derivative of the full oracle's L_adapt (mean of its chunk
    means, 算法 1 with n_u = 1) with respect to the fast MLP's initial
    weights, by central differences, against the meta-gradient of the
    reduced chunk loss fed with the model's own h and r."""
    cfg = MICRO
    w = synth.make_weights(cfg)
    arrays = {k: v.astype(np.float64) for k, v in w.arrays.items()}
    toks = synth.tokens(cfg, cfg.T).astype(np.int64)
    model = O.Model(cfg, arrays)
    top = cfg.n_layers - 1
    names = ("w_gate", "w_up", "w_down")
    W0 = tuple(arrays[f"fast.{top}.{nm}"] for nm in names)
    h, r, tgt = _inputs_of_the_last_block(model, toks, cfg.b)
    grad, L, rows = M.meta_grad_top_mlp(h, r, tgt, W0, model["final_norm"], model["lm_head"], cfg.eta,
                                        cfg.norm_eps, cfg.b)
    res = O.prefill(model, toks)
    assert abs(L - float(np.mean(res.chunk_mean))) <= 1e-12
    assert np.allclose(rows, res.losses, rtol=1e-12, atol=1e-12, equal_nan=True)

    def L_of(Wv):
        a2 = dict(arrays)
        for nm, x in zip(names, Wv):
            a2[f"fast.{top}.{nm}"] = x
        return float(np.mean(O.prefill(O.Model(cfg, a2), toks).chunk_mean))

    for s in range(2):
        v = _rand_dir(W0, 30 + s)
        fd = _fd(L_of, W0, v)
        assert abs(fd - _dot(grad, v)) <= 1e-7 * max(1.0, abs(fd))


# --- planted mistakes: each must fail one of the pins above -----------------


def _mutant_hvp_drops_silu2(orig):
    def f(fw, bw, W, gf, head, eps, V):
        fw = dict(fw, d2=np.zeros_like(fw["d2"]))
        return orig(fw, bw, W, gf, head, eps, V)
    return f


def _mutant_hvp_drops_norm_tangent(orig):
    def f(fw, bw, W, gf, head, eps, V):
        # treat the norm's scale as constant along V
        x = fw["x"]
        fw2 = dict(fw, x=np.zeros_like(x))
        out = orig(fw2, bw, W, gf, head, eps, V)
        return out
    return f


def _mutant_meta_uses_next_weights(orig):
    def f(n_chunks, W0, eta, loss_grad, hvp):
        traj, losses = M.inner_loop(n_chunks, W0, eta, loss_grad)
        u = None
        for c in range(n_chunks - 1, -1, -1):
            _, g = loss_grad(c, traj[c])
            if u is None:
                u = tuple(gi / n_chunks for gi in g)
            else:
                Wn = traj[c + 1]  # Hessian taken after the update instead of before
                u = M._axpy(M._axpy(u, -eta, hvp(c, Wn, u)), 1.0 / n_chunks, g)
        return u, float(np.mean(losses)), losses
    return f


def _mutant_meta_forgets_mean(orig):
    def f(n_chunks, W0, eta, loss_grad, hvp):
        u, L, losses = orig(n_chunks, W0, eta, loss_grad, hvp)
        return tuple(x * n_chunks for x in u), L, losses
    return f


@pytest.mark.parametrize("target,mutant", [
    ("chunk_hvp", _mutant_hvp_drops_silu2),
    ("chunk_hvp", _mutant_hvp_drops_norm_tangent),
    ("meta_grad", _mutant_meta_uses_next_weights),
    ("meta_grad", _mutant_meta_forgets_mean),
])
def test_planted_mistakes_are_caught(monkeypatch, target, mutant):
    orig = getattr(M, target)
    monkeypatch.setattr(M, target, mutant(orig))
    pins = [test_hvp_matches_finite_differences_of_the_gradient, test_hvp_is_symmetric,
            lambda: test_meta_grad_matches_finite_differences_of_the_adapted_loss(0.3),
            test_matrix_quadratic_against_the_explicit_jacobian_product, test_scalar_quadratic_eq8_closed_form]
    caught = False
    for pin in pins:
        try:
            pin()
        except AssertionError:
            caught = True
            break
    assert caught, f"no pin caught the mutation of {target}"


# --- the whole model: fast MLPs in two blocks (Hessian-vector products through SWA)

MICRO2 = MICRO.with_(n_updated=2, eta=0.8)


def _micro2(gains=True):
    cfg = MICRO2
    w = synth.make_weights(cfg)
    arrays = {k: v.astype(np.float64) for k, v in w.arrays.items()}
    if gains:  # norm gains away from 1, so that a gain on the wrong tensor shows
        rng = np.random.default_rng(11)
        for k in arrays:
            if k.endswith("norm"):
                arrays[k] = 1.0 + 0.3 * rng.standard_normal(arrays[k].shape)
    toks = synth.tokens(cfg, cfg.T).astype(np.int64)
    return cfg, O.Model(cfg, arrays), arrays, toks


def _chunk_at(model, toks, c):
    """State and fast weights when chunk c starts (the inner loop run up to it)."""
    res = O.prefill(model, toks, n_chunks=c, keep_state=True) if c else None
    state = res.state if c else O.State(model.cfg, len(toks))
    W = res.W if c else O.init_fast(model)
    return state, W


def _fwd(model, state, W, toks, c):
    import copy
    b = model.cfg.b
    p0 = c * b
    tgt = M._chunk_targets(toks, p0, b)
    _, fwd = O.forward_chunk(model, W, copy.deepcopy(state), toks[p0:p0 + b], p0, tgt)
    nc = int((tgt >= 0).sum())
    return fwd, np.where(tgt >= 0, 1.0 / nc, 0.0)


def _wdir(W, seed):
    rng = np.random.default_rng(seed)
    return {l: {nm: rng.standard_normal(a.shape) for nm, a in W[l].items()} for l in W}


def _wax(W, t, V):
    return {l: {nm: W[l][nm] + t * V[l][nm] for nm in W[l]} for l in W}


def test_model_gradient_repeats_the_inner_loop_backward():
    cfg, model, _, toks = _micro2()
    state, W = _chunk_at(model, toks, 2)
    fwd, wts = _fwd(model, state, W, toks, 2)
    G, _ = M.model_chunk_grad_hvp(model, W, fwd, wts, _wdir(W, 1))
    want = O.backward_chunk(model, W, fwd, wts)
    for l in want:
        for nm in want[l]:
            assert np.abs(G[l][nm] - want[l][nm]).max() <= 1e-13 * np.abs(want[l][nm]).max()


@pytest.mark.parametrize("c", [0, 2])
def test_model_hvp_matches_finite_differences_of_the_gradient(c):
    """Through both blocks (the lower fast MLP reaches the loss through the
    upper block's attention), cached keys held."""
    cfg, model, _, toks = _micro2()
    state, W = _chunk_at(model, toks, c)
    fwd, wts = _fwd(model, state, W, toks, c)
    V = _wdir(W, 2)
    _, HV = M.model_chunk_grad_hvp(model, W, fwd, wts, V)

    def grad(Wx):
        f, w = _fwd(model, state, Wx, toks, c)
        return O.backward_chunk(model, Wx, f, w)

    e = 1e-4
    gs = {t: grad(_wax(W, t, V)) for t in (-2 * e, -e, e, 2 * e)}
    for l in W:
        for nm in W[l]:
            fd = (8.0 * (gs[e][l][nm] - gs[-e][l][nm]) - (gs[2 * e][l][nm] - gs[-2 * e][l][nm])) / (12 * e)
            assert np.abs(HV[l][nm] - fd).max() <= 1e-6 * np.abs(fd).max()


def test_model_hvp_is_symmetric():
    cfg, model, _, toks = _micro2()
    state, W = _chunk_at(model, toks, 1)
    fwd, wts = _fwd(model, state, W, toks, 1)
    U, V = _wdir(W, 3), _wdir(W, 4)
    _, HU = M.model_chunk_grad_hvp(model, W, fwd, wts, U)
    _, HV = M.model_chunk_grad_hvp(model, W, fwd, wts, V)
    a = sum(float(np.sum(V[l][nm] * HU[l][nm])) for l in W for nm in W[l])
    b = sum(float(np.sum(U[l][nm] * HV[l][nm])) for l in W for nm in W[l])
    assert abs(a - b) <= 1e-11 * max(1.0, abs(a))


def test_model_meta_grad_matches_finite_differences_with_the_cache_held():
    """eq. (7) over the model's four chunks against central differences of L
    with every chunk's earlier keys and values held at the unperturbed run's;
    and L itself against the inner loop's own chunk means."""
    cfg, model, arrays, toks = _micro2()
    grad, L, _ = M.meta_grad_model(model, toks)
    base = O.prefill(model, toks, keep_state=True)
    assert abs(L - float(np.mean(base.chunk_mean))) <= 1e-12
    W0 = O.init_fast(model)
    assert abs(M.frozen_adapted_loss(model, toks, W0, base.state) - L) <= 1e-12
    for s in range(2):
        V = _wdir(W0, 40 + s)
        f = lambda t: M.frozen_adapted_loss(model, toks, _wax(W0, t, V), base.state)
        e = 1e-4
        fd = (8.0 * (f(e) - f(-e)) - (f(2 * e) - f(-2 * e))) / (12 * e)
        dot = sum(float(np.sum(grad[l][nm] * V[l][nm])) for l in W0 for nm in W0[l])
        assert abs(fd - dot) <= 1e-7 * max(1.0, abs(fd))
    # neither check is vacuous here: the Hessian term moves the result, and the
    # path through the cached keys (left out by eq. (7)) moves the full L
    no_h = M.meta_grad(4, M._flat(W0), cfg.eta, *_model_closures(model, toks, hessian=False))[0]
    g = M._flat(grad)
    assert max(np.abs(a - c).max() / np.abs(a).max() for a, c in zip(g, no_h)) > 0.1

    def L_full(Wx):
        a2 = dict(arrays)
        for l in Wx:
            for nm in Wx[l]:
                a2[f"fast.{l}.{nm}"] = Wx[l][nm]
        return float(np.mean(O.prefill(O.Model(cfg, a2), toks).chunk_mean))

    V = _wdir(W0, 40)
    e = 1e-4
    f = lambda t: L_full(_wax(W0, t, V))
    fd_full = (8.0 * (f(e) - f(-e)) - (f(2 * e) - f(-2 * e))) / (12 * e)
    dot = sum(float(np.sum(grad[l][nm] * V[l][nm])) for l in W0 for nm in W0[l])
    assert abs(fd_full - dot) > 0.05 * abs(fd_full)


def _model_closures(model, toks, hessian=True):
    """loss_grad / hvp of meta_grad_model, with the Hessian term optionally
    left out (H v = 0)."""
    b = model.cfg.b
    like = O.init_fast(model)
    state = O.State(model.cfg, len(toks))

    def fwd_of(c, Wt):
        tgt = M._chunk_targets(toks, c * b, b)
        loss, fwd = O.forward_chunk(model, M._unflat(Wt, like), state, toks[c * b:(c + 1) * b], c * b, tgt)
        nc = int((tgt >= 0).sum())
        return loss, fwd, np.where(tgt >= 0, 1.0 / nc, 0.0)

    def lg(c, Wt):
        loss, fwd, w = fwd_of(c, Wt)
        return float(np.nanmean(loss)), M._flat(O.backward_chunk(model, M._unflat(Wt, like), fwd, w))

    def hv(c, Wt, v):
        if not hessian:
            return tuple(np.zeros_like(x) for x in v)
        _, fwd, w = fwd_of(c, Wt)
        return M._flat(M.model_chunk_grad_hvp(model, M._unflat(Wt, like), fwd, w, M._unflat(v, like))[1])

    return lg, hv


def test_model_meta_grad_with_one_fast_block_is_the_last_block_case():
    cfg = MICRO
    w = synth.make_weights(cfg)
    arrays = {k: v.astype(np.float64) for k, v in w.arrays.items()}
    toks = synth.tokens(cfg, cfg.T).astype(np.int64)
    model = O.Model(cfg, arrays)
    grad, L, _ = M.meta_grad_model(model, toks)
    top = cfg.n_layers - 1
    W0 = tuple(arrays[f"fast.{top}.{nm}"] for nm in ("w_gate", "w_up", "w_down"))
    h, r, tgt = _inputs_of_the_last_block(model, toks, cfg.b)
    want, L2, _ = M.meta_grad_top_mlp(h, r, tgt, W0, model["final_norm"], model["lm_head"], cfg.eta,
                                      cfg.norm_eps, cfg.b)
    assert abs(L - L2) <= 1e-12
    for nm, w_ in zip(("w_gate", "w_up", "w_down"), want):
        assert np.abs(grad[top][nm] - w_).max() <= 1e-12 * np.abs(w_).max()


# --- op level: the attention tangents a GPU kernel would be checked against


def _swa_case(seed=12, n=5, m=9, H=2, hd=8, k=4):
    rng = np.random.default_rng(seed)
    q, K, V = (rng.standard_normal(s) for s in ((n, H, hd), (m, H, hd), (m, H, hd)))
    qt, Kt, Vt = (rng.standard_normal(s) for s in ((n, H, hd), (m, H, hd), (m, H, hd)))
    do, dot = rng.standard_normal((n, H, hd)), rng.standard_normal((n, H, hd))
    qpos = np.arange(m - n, m)   # the chunk's queries are the last n key positions
    kpos = np.arange(m)
    return q, K, V, qt, Kt, Vt, do, dot, qpos, kpos, k


def test_swa_tangent_matches_finite_differences():
    q, K, V, qt, Kt, Vt, _, _, qpos, kpos, k = _swa_case()
    o_of = lambda t: O.swa(q + t * qt, K + t * Kt, V + t * Vt, qpos, kpos, k)[0]
    _, P = O.swa(q, K, V, qpos, kpos, k)
    _, ot = M.swa_tangent(q, K, V, P, qt, Kt, Vt)
    e = 1e-4
    fd = (8.0 * (o_of(e) - o_of(-e)) - (o_of(2 * e) - o_of(-2 * e))) / (12 * e)
    assert np.abs(ot - fd).max() <= 1e-8 * np.abs(fd).max()


def test_swa_bwd_tangent_matches_finite_differences():
    q, K, V, qt, Kt, Vt, do, dot, qpos, kpos, k = _swa_case(seed=13)
    hd = q.shape[-1]

    def grads(t):
        qq, KK, VV = q + t * qt, K + t * Kt, V + t * Vt
        _, P = O.swa(qq, KK, VV, qpos, kpos, k)
        return O.swa_bwd(do + t * dot, qq, KK, VV, P, hd)

    _, P = O.swa(q, K, V, qpos, kpos, k)
    Pt, _ = M.swa_tangent(q, K, V, P, qt, Kt, Vt)
    tang = M.swa_bwd_tangent(do, dot, q, K, V, P, qt, Kt, Vt, Pt)
    e = 1e-4
    gs = {t: grads(t) for t in (-2 * e, -e, e, 2 * e)}
    for i, a in enumerate(tang):
        fd = (8.0 * (gs[e][i] - gs[-e][i]) - (gs[2 * e][i] - gs[-2 * e][i])) / (12 * e)
        assert np.abs(a - fd).max() <= 1e-8 * np.abs(fd).max()
