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

``chunk_bwd_head`` computes the same gradients by the chunk-parallel WY/UT algebra (real and
rotation decay), the form a backward kernel takes; the tests hold it to the token-level sweep.
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


def l2_normalise_bwd(x, gy):
    """Gradient with respect to x of y = x / sqrt(sum x^2 + eps) over the last axis (the
    normalisation of ``oracle.l2_normalise``), given gy = dL/dy:
    dL/dx = (gy - y (y . gy)) / sqrt(sum x^2 + eps)."""
    from . import L2NORM_EPS
    x = np.asarray(x, dtype=np.float64)
    r = 1.0 / np.sqrt(np.sum(x * x, axis=-1, keepdims=True) + L2NORM_EPS)
    y = x * r
    return (gy - y * np.sum(y * gy, axis=-1, keepdims=True)) * r


def gdr_bwd(q, k, v, g, beta, theta=None, S0=None, gO=None, gS=None, gate_mode=0, scale=1.0, w=None,
            qk_l2norm=False):
    """Whole-batch gradients, head by head (layouts as ``oracle.gdr_fwd``; gO like o, gS like
    S_T).  Returns (o, S_T, grads) with grads a dict of arrays shaped like the inputs
    ("q", "k", "v", "g", "beta", "w" or None, "theta" or None, "S0").  With qk_l2norm, q and k
    are L2-normalised per token and head first (as ``oracle.gdr_fwd`` does), and their gradients
    are taken through the normalisation."""
    f = lambda a: None if a is None else np.asarray(a, dtype=np.float64)
    q, k, v, g, beta, theta, S0, gO, gS, w = map(f, (q, k, v, g, beta, theta, S0, gO, gS, w))
    if qk_l2norm:
        from . import l2_normalise
        o, S_T, out = gdr_bwd(l2_normalise(q), l2_normalise(k), v, g, beta, theta, S0, gO, gS, gate_mode,
                              scale, w)
        out["q"] = l2_normalise_bwd(q, out["q"])
        out["k"] = l2_normalise_bwd(k, out["k"])
        return o, S_T, out
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


def _to_c(x):
    """Key pairs (2j, 2j+1) of the last axis as complex numbers x_2j + i x_2j+1."""
    return x[..., 0::2] + 1j * x[..., 1::2]


def _to_r(z):
    """Inverse of ``_to_c``."""
    x = np.empty(z.shape[:-1] + (2 * z.shape[-1],))
    x[..., 0::2], x[..., 1::2] = z.real, z.imag
    return x


def chunk_bwd_head(q, k, v, g, beta, S0, gO, gS, gate_mode, scale, w, chunk=64, theta=None):
    """The same gradients for one head, by the chunk-parallel WY/UT algebra that a backward
    kernel follows, restated in fp64 ("CARVE" page, section 1 item 3: the WY-form chunk
    solver; "Semidirect Fourier Delta Attention" page, *Constructive Chunk-WY Theorem*).

    Forward of a chunk with start state S0 (dv x dk), gamma = in-chunk cumulative log decay:
        Ktil = K e^{gamma},  Qtil = scale Q e^{gamma},  Khat = K e^{-gamma},  Kdec = K e^{gamma_L - gamma}
        A = diag(beta) strict_lower(Ktil Khat^T),  P = incl_lower(Qtil Khat^T),  T = (I + A)^{-1}
        R = diag(w) V - diag(beta) Ktil S0^T,  E = T R
        O = Qtil S0^T + P E,  S_L = S0 diag(e^{gamma_L}) + E^T Kdec
    Rotation (theta given): with key pairs as complex numbers and the cumulative factor
    Lam_r = prod over the chunk's tokens t <= r of alpha_t e^{i theta_t} (per pair), the same
    algebra holds with Ktil = K conj(Lam), Qtil = scale Q conj(Lam), Khat = K / Lam,
    Kdec = K Lam_L / Lam and S0 Lam_L, every product of two tiles being the real dot product
    of their (re, im) pairs.  The chunk-start states come from a forward sweep; the backward
    sweep runs the chunks in reverse with dS_L of chunk c = dS0 of chunk c + 1 (gS for the
    last chunk).  Returns (o, S_T, grads) like ``gdr_bwd_head``.
    """
    T_, dk = q.shape
    dv = v.shape[1]
    rot = theta is not None
    wv = beta if w is None else w
    nc = (T_ + chunk - 1) // chunk
    al, dal = _alpha(g, gate_mode)
    lg = np.log(al)            # log alpha per token and key dim (rotation: per pair)
    dlg = dal / al             # d log alpha / d (gate input)

    def parts(c, S0c):
        t0, t1 = c * chunk, min((c + 1) * chunk, T_)
        K, Q, V = k[t0:t1], q[t0:t1], v[t0:t1]
        f = dict(t0=t0, t1=t1, K=K, Q=Q, V=V, S0=S0c)
        if not rot:
            gam = np.cumsum(lg[t0:t1], axis=0)
            gl = gam[-1]
            Kt, Qt, Kh, Kd = K * np.exp(gam), scale * Q * np.exp(gam), K * np.exp(-gam), K * np.exp(gl - gam)
            S0dec = S0c * np.exp(gl)[None, :]
            f.update(gam=gam, gl=gl)
        else:
            Lam = np.exp(np.cumsum(lg[t0:t1] + 1j * theta[t0:t1], axis=0))
            LamL = Lam[-1]
            Kc, Qc = _to_c(K), _to_c(Q)
            Kt, Qt = _to_r(Kc * np.conj(Lam)), _to_r(scale * Qc * np.conj(Lam))
            Kh, Kd = _to_r(Kc / Lam), _to_r(Kc * LamL / Lam)
            S0dec = _to_r(_to_c(S0c) * LamL[None, :])
            f.update(Lam=Lam, LamL=LamL, Kc=Kc, Qc=Qc)
        L = t1 - t0
        Ms, Mi = np.tril(np.ones((L, L)), -1), np.tril(np.ones((L, L)))
        Ap = Kt @ Kh.T
        A = beta[t0:t1, None] * (Ap * Ms)
        P = (Qt @ Kh.T) * Mi
        Tm = np.linalg.inv(np.eye(L) + A)
        R = wv[t0:t1, None] * V - beta[t0:t1, None] * (Kt @ S0c.T)
        E = Tm @ R
        O = Qt @ S0c.T + P @ E
        SL = S0dec + E.T @ Kd
        f.update(Kt=Kt, Qt=Qt, Kh=Kh, Kd=Kd, Ms=Ms, Mi=Mi, Ap=Ap, P=P, Tm=Tm, R=R, E=E, O=O, SL=SL)
        return f

    S = np.zeros((dv, dk)) if S0 is None else np.array(S0, dtype=np.float64)
    fw = []
    o = np.zeros((T_, dv))
    for c in range(nc):
        f = parts(c, S)
        fw.append(f)
        o[f["t0"]:f["t1"]] = f["O"]
        S = f["SL"]
    grads = {"q": np.zeros_like(q), "k": np.zeros_like(k), "v": np.zeros_like(v), "g": np.zeros_like(g),
             "beta": np.zeros(T_), "w": None if w is None else np.zeros(T_),
             "theta": np.zeros_like(theta) if rot else None}
    dSL = np.zeros((dv, dk)) if gS is None else np.array(gS, dtype=np.float64)
    for c in range(nc - 1, -1, -1):
        f = fw[c]
        t0, t1 = f["t0"], f["t1"]
        dO = np.zeros((t1 - t0, dv)) if gO is None else gO[t0:t1]
        S0c, E, P, Tm, R = f["S0"], f["E"], f["P"], f["Tm"], f["R"]
        Kt, Qt, Kh, Kd, K = f["Kt"], f["Qt"], f["Kh"], f["Kd"], f["K"]
        bt = beta[t0:t1]
        # outputs: O = Qtil S0^T + P E ;  S_L = (S0 decayed over the chunk) + E^T Kdec
        dE = P.T @ dO + Kd @ dSL.T
        dP = (dO @ E.T) * f["Mi"]
        dQt = dO @ S0c + dP @ Kh
        dKh = dP.T @ Qt
        dS0 = dO.T @ Qt
        dKd = E @ dSL
        # E = T R ;  T = (I + A)^{-1}
        dR = Tm.T @ dE
        dA = -Tm.T @ (dE @ R.T) @ Tm.T
        # R = diag(w) V - diag(beta) Ktil S0^T
        grads["v"][t0:t1] = wv[t0:t1, None] * dR
        KS = Kt @ S0c.T
        dbeta = -np.sum(dR * KS, axis=1)
        if w is None:
            dbeta += np.sum(dR * f["V"], axis=1)
        else:
            grads["w"][t0:t1] = np.sum(dR * f["V"], axis=1)
        dKt = -(bt[:, None] * dR) @ S0c
        dS0 -= (bt[:, None] * dR).T @ Kt
        # A = diag(beta) strict_lower(Ktil Khat^T)
        dbeta += np.sum(dA * f["Ap"] * f["Ms"], axis=1)
        dAp = bt[:, None] * dA * f["Ms"]
        dKt += dAp @ Kh
        dKh += dAp.T @ Kt
        grads["beta"][t0:t1] = dbeta
        # factors of K and Q, the chunk's decay of S0, and the cumulative decay
        if not rot:
            gam, gl = f["gam"], f["gl"]
            eg = np.exp(gam)
            dS0 += dSL * np.exp(gl)[None, :]
            grads["q"][t0:t1] = scale * dQt * eg
            grads["k"][t0:t1] = dKt * eg + dKh / eg + dKd * np.exp(gl - gam)
            dgam = dKt * Kt + dQt * Qt - dKh * Kh - dKd * Kd
            dgam[-1] += np.exp(gl) * np.sum(S0c * dSL, axis=0) + np.sum(dKd * Kd, axis=0)   # gamma_L terms
            dlog = np.cumsum(dgam[::-1], axis=0)[::-1]          # gamma = cumsum(log alpha)
            grads["g"][t0:t1] = dlog * dlg[t0:t1]
        else:
            # complex gradients g_z with dL = Re(conj(g_z) dz) per pair
            Lam, LamL, Kc, Qc = f["Lam"], f["LamL"], f["Kc"], f["Qc"]
            gKt, gQt, gKh, gKd, gSL = _to_c(dKt), _to_c(dQt), _to_c(dKh), _to_c(dKd), _to_c(dSL)
            dS0 += _to_r(gSL * np.conj(LamL)[None, :])
            grads["q"][t0:t1] = _to_r(scale * gQt * Lam)
            grads["k"][t0:t1] = _to_r(gKt * Lam + gKh * np.conj(1.0 / Lam) + gKd * np.conj(LamL / Lam))
            gLam = (np.conj(gKt) * Kc + scale * np.conj(gQt) * Qc - gKh * np.conj(Kc / Lam ** 2)
                    - gKd * np.conj(Kc * LamL / Lam ** 2))
            gLam[-1] += np.sum(gKd * np.conj(Kc / Lam), axis=0) + np.sum(gSL * np.conj(_to_c(S0c)), axis=0)
            gz = np.cumsum((gLam * np.conj(Lam))[::-1], axis=0)[::-1]   # Lam = exp(cumsum(log alpha + i theta))
            grads["g"][t0:t1] = gz.real * dlg[t0:t1]
            grads["theta"][t0:t1] = gz.imag
        dSL = dS0
    grads["S0"] = dSL
    return o, S, grads
