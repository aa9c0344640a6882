"""fp64 reverse-mode gradients of the token recurrence: the oracle of a backward pass.

TEST INFRASTRUCTURE ONLY, like the rest of ``oracle/``: imported by tests/, never by the
product path.

The forward is the token step of ``gdr_oracle.c``, per head, with the state S (dv x dk) and
row vectors ("Semidirect Fourier Delta Attention" page, section *Core architecture*: decay,
then erase along k_t, then write; "CARVE" page, sections 2.1-2.2: erase strength beta_t and
write strength w_t):

    X_t = S_{t-1} D_t,   e_t = w_t v_t - beta_t X_t k_t,   S_t = X_t + e_t k_t^T,
    o_t = S_t (scale q_t)

with D_t = diag(alpha_t), alpha_t = exp(g_t) (gate mode 0) or sigmoid(-a_t) = exp(-softplus(a_t))
(gate mode 1); in rotation mode each key pair (2j, 2j+1) of a row is the complex number
x + i y, multiplied by alpha_{t,j} e^{i theta_{t,j}}.

Given gO = dL/do [B,T,H,dv] and gS = dL/dS_T [B,H,dv,dk] (either may be None: zero), the
chain rule runs backwards over the tokens with the states recomputed forward and kept
(T x dv x dk doubles per head, for small problems):

    G <- G + gO_t (scale q_t)^T                         (G = dL/dS_t)
    dq_t = scale S_t^T gO_t
    ge = G k_t;  dk_t = G^T e_t - beta_t X_t^T ge;  dv_t = w_t ge
    dw_t = ge . v_t;  dbeta_t = -ge . (X_t k_t)          (tied: w = beta, the two add)
    gX = G - beta_t ge k_t^T
    G <- gX D_t^T  (rotation: gX times alpha e^{-i theta} per pair);  dS0 = G after token 1
    dalpha = sum over rows of gX * dX/dalpha;  dtheta = sum over rows of (gX_b X_a - gX_a X_b)
    dg = dalpha * dalpha/dg  (alpha for gate mode 0; -alpha sigmoid(a) for gate mode 1)
"""
import numpy as np


def _alpha(g_in, gate_mode):
    """alpha and d alpha / d (gate input), elementwise."""
    g_in = np.asarray(g_in, dtype=np.float64)
    if gate_mode == 1:
        sp = np.maximum(g_in, 0.0) + np.log1p(np.exp(-np.abs(g_in)))    # softplus(a)
        al = np.exp(-sp)
        return al, -al / (1.0 + np.exp(-g_in))                          # d/da exp(-softplus a)
    al = np.exp(g_in)
    return al, al


def _decay(S, al, c, s):
    """X = S D for real (c is None) or rotation decay."""
    if c is None:
        return S * al[None, :]
    x, y = S[:, 0::2], S[:, 1::2]
    X = np.empty_like(S)
    X[:, 0::2] = al * (c * x - s * y)
    X[:, 1::2] = al * (s * x + c * y)
    return X


def gdr_bwd_head(q, k, v, g, beta, theta, S0, gO, gS, gate_mode, scale, w):
    """One head: q, k [T,dk]; v [T,dv]; g [T,ng]; beta, w [T] (w may be None); theta [T,dk/2]
    or None; S0, gS [dv,dk] or None; gO [T,dv] or None.  Returns (o, S_T, grads)."""
    T, dk = q.shape
    dv = v.shape[1]
    rot = theta is not None
    tied = w is None
    wv = beta if tied else w
    S = np.zeros((dv, dk)) if S0 is None else np.array(S0, dtype=np.float64)
    prev, Xs, es, Ss, als, dals = [], [], [], [], [], []
    o = np.zeros((T, dv))
    for t in range(T):
        al, dal = _alpha(g[t], gate_mode)
        c = np.cos(theta[t]) if rot else None
        s_ = np.sin(theta[t]) if rot else None
        X = _decay(S, al, c, s_)
        e = wv[t] * v[t] - beta[t] * (X @ k[t])
        prev.append(S)
        S = X + np.outer(e, k[t])
        o[t] = S @ (scale * q[t])
        Xs.append(X); es.append(e); Ss.append(S); als.append(al); dals.append(dal)
    grads = {n: np.zeros_like(a) for n, a in (("q", q), ("k", k), ("v", v), ("g", g))}
    grads["beta"] = np.zeros(T)
    grads["w"] = None if tied else np.zeros(T)
    grads["theta"] = np.zeros_like(theta) if rot else None
    G = np.zeros((dv, dk)) if gS is None else np.array(gS, dtype=np.float64)
    for t in range(T - 1, -1, -1):
        X, e, St, Sp, al, dal = Xs[t], es[t], Ss[t], prev[t], als[t], dals[t]
        if gO is not None:
            G = G + np.outer(gO[t], scale * q[t])
            grads["q"][t] = scale * (St.T @ gO[t])
        ge = G @ k[t]
        xk = X @ k[t]
        grads["k"][t] = G.T @ e - beta[t] * (X.T @ ge)
        grads["v"][t] = wv[t] * ge
        if tied:
            grads["beta"][t] = ge @ v[t] - ge @ xk
        else:
            grads["beta"][t] = -(ge @ xk)
            grads["w"][t] = ge @ v[t]
        gX = G - beta[t] * np.outer(ge, k[t])
        if not rot:
            galpha = np.sum(gX * Sp, axis=0)
            G = gX * al[None, :]
        else:
            c, s_ = np.cos(theta[t]), np.sin(theta[t])
            ga, gb = gX[:, 0::2], gX[:, 1::2]
            x, y = Sp[:, 0::2], Sp[:, 1::2]
            galpha = np.sum(ga * (c * x - s_ * y) + gb * (s_ * x + c * y), axis=0)
            grads["theta"][t] = np.sum(gb * X[:, 0::2] - ga * X[:, 1::2], axis=0)
            G = np.empty_like(gX)
            G[:, 0::2] = al * (c * ga + s_ * gb)
            G[:, 1::2] = al * (c * gb - s_ * ga)
        grads["g"][t] = galpha * dal
    grads["S0"] = G
    return o, S, grads


def gdr_bwd(q, k, v, g, beta, theta=None, S0=None, gO=None, gS=None, gate_mode=0, scale=1.0, w=None):
    """Whole-batch gradients, head by head (layouts as ``oracle.gdr_fwd``; gO like o, gS like
    S_T).  Returns (o, S_T, grads) with grads a dict of arrays shaped like the inputs
    ("q", "k", "v", "g", "beta", "w" or None, "theta" or None, "S0")."""
    f = lambda a: None if a is None else np.asarray(a, dtype=np.float64)
    q, k, v, g, beta, theta, S0, gO, gS, w = map(f, (q, k, v, g, beta, theta, S0, gO, gS, w))
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    o = np.zeros((B, T, H, dv))
    S_T = np.zeros((B, H, dv, dk))
    out = {"q": np.zeros_like(q), "k": np.zeros_like(k), "v": np.zeros_like(v), "g": np.zeros_like(g),
           "beta": np.zeros_like(beta), "w": None if w is None else np.zeros_like(w),
           "theta": None if theta is None else np.zeros_like(theta), "S0": np.zeros((B, H, dv, dk))}
    for b in range(B):
        for h in range(H):
            sel = lambda a: None if a is None else a[b, :, h]
            oh, Sh, gr = gdr_bwd_head(sel(q), sel(k), sel(v), sel(g), sel(beta), sel(theta),
                                      None if S0 is None else S0[b, h], sel(gO),
                                      None if gS is None else gS[b, h], gate_mode, scale, sel(w))
            o[b, :, h] = oh
            S_T[b, h] = Sh
            for n in ("q", "k", "v", "g", "beta", "w", "theta"):
                if out[n] is not None:
                    out[n][b, :, h] = gr[n]
            out["S0"][b, h] = gr["S0"]
    return o, S_T, out
