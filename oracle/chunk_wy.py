"""fp64 numpy restatements of the chunk-parallel algebra, for one head.

TEST INFRASTRUCTURE ONLY (see ``oracle/__init__``).  These are checked against the
token-by-token recurrence in ``gdr_oracle.c``; they are not used by the product.

Two forms are given, both with explicit d x d matrices so that each step can be
read against the pages:

``sfda_chunk_wy`` -- the constructive chunk-WY theorem of the "Semidirect Fourier
    Delta Attention" page (section "Constructive Chunk-WY Theorem") and its
    exact affine chunk transfer (section "Main contributions").  In the page's
    orientation the state Z = S^T is dk x dv and a token acts as
    Z_t = A_t Z_{t-1} + u_t v_t^T with A_t = Lambda_t - u_t r_t^T,
    u_t = beta_t k_t, r_t = Lambda_t^T k_t.  The product P_t = A_t ... A_1 is kept
    as Gamma_t - Y_t M_t W_t^T with Y_t, W_t of size d x t and M_t lower
    triangular t x t, grown left to right inside the chunk and reset at its end;
    the write summary B_chunk comes from the same recursion started at Z = 0,
    and the boundary state is Z_end = P_C Z_start + B_C.

``ut_chunk`` -- the UT-transform form that the CUDA kernels evaluate (the WY
    triangular chunk solver of the "CARVE" page, section 1 item 3 and
    section 3 item 1).  With P_r = D_1 ... D_r (our orientation, D_t = Lambda_t^T):
        Ktil_r = P_r k_r,  Khat_i = P_i^{-T} k_i,  Kdec_i = P_C^T P_i^{-T} k_i,
        Qtil_r = P_r q_r,
        A[r,i]  = beta_r Khat_i . Ktil_r   (i < r),   Pm[r,i] = Khat_i . Qtil_r  (i <= r)
        Tm = (I + A)^{-1},  U = Tm diag(beta) V,  Wk = Tm diag(beta) Ktil
        E  = U - Wk S_0^T        (the chunk's pseudo-values)
        O  = Qtil S_0^T + Pm E
        S_C = S_0 P_C + E^T Kdec
"""
import numpy as np

GATE_LOGDECAY = 0
GATE_NEG_SOFTPLUS = 1


def log_decay(g, gate_mode):
    g = np.asarray(g, dtype=np.float64)
    if gate_mode == GATE_NEG_SOFTPLUS:
        return -np.logaddexp(0.0, g)   # -softplus(a)
    return g


def decay_matrix(g_t, theta_t, dk, gate_mode):
    """D_t (dk x dk) acting on the right of S (dv x dk).

    Real mode: diag(exp(g_t)).  Rotation mode: 2x2 blocks alpha [[c, s], [-s, c]],
    so that the key pair (x, y) of a row of S goes to alpha e^{i theta} (x + i y);
    this is Lambda_t^T for the page's Lambda_t = diag(alpha e^{i theta}).
    """
    lg = log_decay(g_t, gate_mode)
    if theta_t is None:
        return np.diag(np.exp(lg))
    D = np.zeros((dk, dk))
    for j in range(dk // 2):
        a = np.exp(lg[j])
        c, s = np.cos(theta_t[j]), np.sin(theta_t[j])
        D[2 * j, 2 * j] = a * c
        D[2 * j, 2 * j + 1] = a * s
        D[2 * j + 1, 2 * j] = -a * s
        D[2 * j + 1, 2 * j + 1] = a * c
    return D


def _chunks(T, C):
    return [(s, min(s + C, T)) for s in range(0, T, C)]


def sfda_chunk_wy(q, k, v, g, beta, theta=None, S0=None, chunk=64,
                  gate_mode=GATE_LOGDECAY, scale=1.0):
    """Single head: q, k [T,dk]; v [T,dv]; g [T,dk or dk/2]; beta [T]; theta [T,dk/2].

    Returns (o [T,dv], S_T [dv,dk]) computed through the constructive chunk-WY
    product and the affine chunk transfer.  Also returns, per chunk, the pair
    (P_C, B_C) so tests can inspect the rank of the correction.
    """
    T, dk = q.shape
    dv = v.shape[1]
    Z = np.zeros((dk, dv)) if S0 is None else np.array(S0, dtype=np.float64).T.copy()
    o = np.zeros((T, dv))
    transfers = []
    for (s, e) in _chunks(T, chunk):
        Gam = np.eye(dk)
        Y = np.zeros((dk, 0))
        W = np.zeros((dk, 0))
        M = np.zeros((0, 0))
        Bw = np.zeros((dk, dv))            # write summary, zero initial state
        Z0 = Z.copy()
        for t in range(s, e):
            Lam = decay_matrix(g[t], None if theta is None else theta[t], dk, gate_mode).T
            u = beta[t] * k[t]
            r = Lam.T @ k[t]
            m_row = -(r @ Y) @ M if M.size else np.zeros(0)
            n = M.shape[0]
            M_new = np.zeros((n + 1, n + 1))
            M_new[:n, :n] = M
            M_new[n, :n] = m_row
            M_new[n, n] = 1.0
            Y = np.concatenate([Lam @ Y, u[:, None]], axis=1)
            W = np.concatenate([W, (Gam.T @ r)[:, None]], axis=1)
            M = M_new
            Gam = Lam @ Gam
            A_t = Lam - np.outer(u, r)
            Bw = A_t @ Bw + np.outer(u, v[t])
            P_t = Gam - Y @ M @ W.T
            Z_t = P_t @ Z0 + Bw
            o[t] = Z_t.T @ (scale * q[t])
        P_C = Gam - Y @ M @ W.T
        Z = P_C @ Z0 + Bw
        transfers.append((P_C, Gam, Bw))
    return o, Z.T.copy(), transfers


def ut_chunk(q, k, v, g, beta, theta=None, S0=None, chunk=64,
             gate_mode=GATE_LOGDECAY, scale=1.0):
    """Single head, UT-transform chunk solver with explicit P_r matrices.

    Returns (o [T,dv], S_T [dv,dk]).
    """
    T, dk = q.shape
    dv = v.shape[1]
    S = np.zeros((dv, dk)) if S0 is None else np.array(S0, dtype=np.float64).copy()
    o = np.zeros((T, dv))
    for (s, e) in _chunks(T, chunk):
        L = e - s
        P = []
        acc = np.eye(dk)
        for t in range(s, e):
            acc = acc @ decay_matrix(g[t], None if theta is None else theta[t], dk, gate_mode)
            P.append(acc.copy())
        PC = P[-1]
        Kt = np.stack([P[r] @ k[s + r] for r in range(L)])
        Kh = np.stack([np.linalg.solve(P[i].T, k[s + i]) for i in range(L)])
        Kd = Kh @ PC                                   # rows (P_C^T P_i^{-T} k_i)^T
        Qt = np.stack([P[r] @ (scale * q[s + r]) for r in range(L)])
        b = beta[s:e]
        A = np.tril(b[:, None] * (Kt @ Kh.T), -1)      # A[r,i] = beta_r Khat_i . Ktil_r
        Pm = np.tril(Qt @ Kh.T)                        # inclusive of the diagonal
        Tm = np.linalg.inv(np.eye(L) + A)
        U = Tm @ (b[:, None] * v[s:e])
        Wk = Tm @ (b[:, None] * Kt)
        E = U - Wk @ S.T
        o[s:e] = Qt @ S.T + Pm @ E
        S = S @ PC + E.T @ Kd
    return o, S
