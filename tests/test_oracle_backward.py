"""Pins of the fp64 backward oracle (oracle/backward.py) against the forward oracle it
differentiates (the C token recurrence): central finite differences of every input, exact
adjoint identities for the inputs the outputs are linear in, and planted mistakes."""
import numpy as np
import pytest

import oracle
from oracle import backward as bwd


def _problem(rng, T, H, dk, dv, rotation, untied, gate_mode):
    q = rng.standard_normal((1, T, H, dk))
    k = rng.standard_normal((1, T, H, dk))
    k /= np.linalg.norm(k, axis=-1, keepdims=True)
    v = rng.standard_normal((1, T, H, dv))
    ng = dk // 2 if rotation else dk
    g = rng.standard_normal((1, T, H, ng)) if gate_mode == 1 else -np.abs(rng.standard_normal((1, T, H, ng))) * 0.3
    beta = 1.0 / (1.0 + np.exp(-rng.standard_normal((1, T, H))))
    w = rng.uniform(0.2, 1.2, (1, T, H)) if untied else None
    theta = rng.uniform(-np.pi, np.pi, (1, T, H, dk // 2)) if rotation else None
    S0 = rng.standard_normal((1, H, dv, dk)) * 0.5
    return dict(q=q, k=k, v=v, g=g, beta=beta, w=w, theta=theta, S0=S0)


def _loss(x, gO, gS, gate_mode, scale, qk_l2norm=False):
    o, S_T = oracle.gdr_fwd(x["q"], x["k"], x["v"], x["g"], x["beta"], x["theta"], x["S0"],
                            gate_mode=gate_mode, scale=scale, w=x["w"], qk_l2norm=qk_l2norm)
    return float(np.sum(gO * o) + np.sum(gS * S_T))


@pytest.mark.parametrize("rotation,untied,gate_mode", [(False, False, 1), (False, True, 0), (True, False, 0),
                                                       (True, True, 1)])
def test_backward_matches_central_differences(rotation, untied, gate_mode):
    """Every element of every input: (L(x + h) - L(x - h)) / 2h with L = <gO, o> + <gS, S_T>
    computed by the C forward oracle, against the backward oracle's gradient."""
    rng = np.random.default_rng(300 + 2 * rotation + untied)
    T, H, dk, dv, scale = 6, 2, 4, 3, 0.7
    x = _problem(rng, T, H, dk, dv, rotation, untied, gate_mode)
    gO = rng.standard_normal((1, T, H, dv))
    gS = rng.standard_normal((1, H, dv, dk))
    o, S_T, grads = bwd.gdr_bwd(x["q"], x["k"], x["v"], x["g"], x["beta"], x["theta"], x["S0"], gO, gS,
                                gate_mode=gate_mode, scale=scale, w=x["w"])
    o_ref, S_ref = oracle.gdr_fwd(x["q"], x["k"], x["v"], x["g"], x["beta"], x["theta"], x["S0"],
                                  gate_mode=gate_mode, scale=scale, w=x["w"])
    assert np.max(np.abs(o - o_ref)) < 1e-12 and np.max(np.abs(S_T - S_ref)) < 1e-12
    h = 1e-6
    names = ["q", "k", "v", "g", "beta", "S0"] + (["w"] if untied else []) + (["theta"] if rotation else [])
    for n in names:
        fd = np.zeros_like(x[n])
        for idx in np.ndindex(x[n].shape):
            xp = {m: (None if a is None else a.copy()) for m, a in x.items()}
            xm = {m: (None if a is None else a.copy()) for m, a in x.items()}
            xp[n][idx] += h
            xm[n][idx] -= h
            fd[idx] = (_loss(xp, gO, gS, gate_mode, scale) - _loss(xm, gO, gS, gate_mode, scale)) / (2 * h)
        err = np.max(np.abs(grads[n] - fd)) / max(np.max(np.abs(fd)), 1e-12)
        assert err < 1e-6, (n, err)
    assert (grads["w"] is None) == (not untied) and (grads["theta"] is None) == (not rotation)


@pytest.mark.parametrize("rotation", [False, True])
def test_backward_through_the_l2_normalisation_matches_central_differences(rotation):
    """With qk_l2norm the forward oracle normalises q and k itself; the backward oracle's dq and
    dk (through the normalisation) against central differences of that forward, on raw q and k
    of norms far from 1 and one q row near the epsilon's scale."""
    rng = np.random.default_rng(330 + rotation)
    T, H, dk, dv, scale = 5, 1, 4, 3, 0.6
    x = _problem(rng, T, H, dk, dv, rotation, False, 1)
    x["q"] *= 3.0
    x["k"] = x["k"] * rng.uniform(0.2, 4.0, (1, T, H, 1))
    x["q"][0, 2, 0] *= 1e-3                       # |q| ~ 5e-3: the epsilon matters
    gO = rng.standard_normal((1, T, H, dv))
    gS = rng.standard_normal((1, H, dv, dk))
    _, _, grads = bwd.gdr_bwd(x["q"], x["k"], x["v"], x["g"], x["beta"], x["theta"], x["S0"], gO, gS,
                              gate_mode=1, scale=scale, qk_l2norm=True)
    h = 1e-7
    for n in ("q", "k", "beta"):
        fd = np.zeros_like(x[n])
        for idx in np.ndindex(x[n].shape):
            xp = {m: (None if a is None else a.copy()) for m, a in x.items()}
            xm = {m: (None if a is None else a.copy()) for m, a in x.items()}
            xp[n][idx] += h
            xm[n][idx] -= h
            fd[idx] = (_loss(xp, gO, gS, 1, scale, True) - _loss(xm, gO, gS, 1, scale, True)) / (2 * h)
        err = np.max(np.abs(grads[n] - fd)) / max(np.max(np.abs(fd)), 1e-12)
        assert err < 1e-5, (n, err)
    # the un-normalised gradient is a different vector (the pin sees a missing projection)
    _, _, raw = bwd.gdr_bwd(oracle.l2_normalise(x["q"]), oracle.l2_normalise(x["k"]), x["v"], x["g"], x["beta"],
                            x["theta"], x["S0"], gO, gS, gate_mode=1, scale=scale)
    assert np.max(np.abs(raw["k"] - grads["k"])) > 1e-2 * np.max(np.abs(grads["k"]))


def test_backward_adjoint_identities_are_exact():
    """o and S_T are linear in (S0, v): for any direction d, L(x + d) - L(x) equals
    <grad, d> up to rounding, with no finite-difference error."""
    rng = np.random.default_rng(310)
    T, H, dk, dv = 9, 2, 6, 5
    x = _problem(rng, T, H, dk, dv, True, True, 1)
    gO = rng.standard_normal((1, T, H, dv))
    gS = rng.standard_normal((1, H, dv, dk))
    _, _, grads = bwd.gdr_bwd(x["q"], x["k"], x["v"], x["g"], x["beta"], x["theta"], x["S0"], gO, gS,
                              gate_mode=1, w=x["w"])
    L0 = _loss(x, gO, gS, 1, 1.0)
    for n in ("S0", "v"):
        d = rng.standard_normal(x[n].shape)
        xd = dict(x)
        xd[n] = x[n] + d
        assert abs((_loss(xd, gO, gS, 1, 1.0) - L0) - np.sum(grads[n] * d)) < 1e-10 * max(1.0, abs(L0))


def test_backward_catches_planted_mistakes():
    """The finite-difference pin is sharp enough to see plausible mistakes in a backward: the
    erase term's gradient dropped from dk, the rotation's adjoint taken with e^{+i theta}, and
    the readout gradient taken from the pre-update state."""
    rng = np.random.default_rng(320)
    T, H, dk, dv = 5, 1, 4, 3
    x = _problem(rng, T, H, dk, dv, True, False, 0)
    gO = rng.standard_normal((1, T, H, dv))
    gS = rng.standard_normal((1, H, dv, dk))
    sel = lambda a: None if a is None else a[0, :, 0]
    args = (sel(x["q"]), sel(x["k"]), sel(x["v"]), sel(x["g"]), sel(x["beta"]), sel(x["theta"]), x["S0"][0, 0],
            sel(gO), gS[0, 0], 0, 1.0, None)
    _, _, ok = bwd.gdr_bwd_head(*args)

    def fd(n):
        out = np.zeros_like(x[n])
        for idx in np.ndindex(x[n].shape):
            xp = {m: (None if a is None else a.copy()) for m, a in x.items()}
            xm = {m: (None if a is None else a.copy()) for m, a in x.items()}
            xp[n][idx] += 1e-6
            xm[n][idx] -= 1e-6
            out[idx] = (_loss(xp, gO, gS, 0, 1.0) - _loss(xm, gO, gS, 0, 1.0)) / 2e-6
        return out[0, :, 0] if n != "S0" else out[0, 0]

    ref = {n: fd(n) for n in ("k", "q", "S0")}
    for n in ref:
        assert np.max(np.abs(ok[n] - ref[n])) < 1e-6 * np.max(np.abs(ref[n])), n
    q, k, v, g, beta, theta, S0 = args[:7]
    S = S0.copy()                   # forward states X_t of this problem
    Xs = []
    for t in range(T):
        al = np.exp(g[t])
        c, s_ = np.cos(theta[t]), np.sin(theta[t])
        X = bwd._decay(S, al, c, s_)
        Xs.append(X)
        e = beta[t] * (v[t] - X @ k[t])
        S = X + np.outer(e, k[t])

    def back(conj_sign):
        """The state adjoint G = dL/dS_t run backwards; conj_sign = +1 multiplies by
        alpha e^{-i theta} (the adjoint of the decay), -1 by alpha e^{+i theta} (a mistake).
        Returns dS0 and the dk of the correct sweep without the erase term's -beta X^T ge."""
        G = gS[0, 0].copy()
        k_wo = np.zeros_like(k)
        for t in range(T - 1, -1, -1):
            G = G + np.outer(gO[0, t, 0], q[t])
            ge = G @ k[t]
            k_wo[t] = ok["k"][t] + beta[t] * (Xs[t].T @ ge)
            gX = G - beta[t] * np.outer(ge, k[t])
            al = np.exp(g[t])
            c, s_ = np.cos(theta[t]), conj_sign * np.sin(theta[t])
            Gn = np.empty_like(gX)
            Gn[:, 0::2] = al * (c * gX[:, 0::2] + s_ * gX[:, 1::2])
            Gn[:, 1::2] = al * (c * gX[:, 1::2] - s_ * gX[:, 0::2])
            G = Gn
        return G, k_wo

    dS0_ok, bad_k = back(+1)
    assert np.max(np.abs(dS0_ok - ref["S0"])) < 1e-6 * np.max(np.abs(ref["S0"]))     # the sweep is right
    # (a) dk without the erase term's -beta X^T ge
    assert np.max(np.abs(bad_k - ref["k"])) > 1e-3 * np.max(np.abs(ref["k"]))
    # (b) the adjoint of the rotation with e^{+i theta}
    dS0_bad, _ = back(-1)
    assert np.max(np.abs(dS0_bad - ref["S0"])) > 1e-3 * np.max(np.abs(ref["S0"]))
    # (c) dq from the pre-update state S_{t-1}
    S = S0.copy()
    bad_q = np.zeros_like(q)
    for t in range(T):
        bad_q[t] = S.T @ gO[0, t, 0]
        al = np.exp(g[t])
        X = bwd._decay(S, al, np.cos(theta[t]), np.sin(theta[t]))
        S = X + np.outer(beta[t] * (v[t] - X @ k[t]), k[t])
    assert np.max(np.abs(bad_q - ref["q"])) > 1e-3 * np.max(np.abs(ref["q"]))


@pytest.mark.parametrize("T,chunk,untied,gate_mode,rotation", [(70, 16, False, 1, False), (37, 8, True, 0, False),
                                                               (64, 64, True, 1, False), (5, 64, False, 0, False),
                                                               (70, 16, True, 1, True), (37, 8, False, 0, True),
                                                               (3, 64, True, 0, True)])
def test_chunked_backward_equals_the_token_backward(T, chunk, untied, gate_mode, rotation):
    """The chunk-parallel WY/UT restatement of the backward (what a backward kernel computes,
    chunk by chunk with the state gradient carried backwards) against the token-level reverse
    sweep: outputs, final state and every gradient, several chunks and a ragged last one."""
    rng = np.random.default_rng(400 + T)
    dk, dv, scale = 8, 5, 0.8
    x = _problem(rng, T, 1, dk, dv, rotation, untied, gate_mode)
    gO = rng.standard_normal((1, T, 1, dv))
    gS = rng.standard_normal((1, 1, dv, dk))
    sel = lambda a: None if a is None else a[0, :, 0]
    args = (sel(x["q"]), sel(x["k"]), sel(x["v"]), sel(x["g"]), sel(x["beta"]))
    o1, S1, g1 = bwd.gdr_bwd_head(*args, sel(x["theta"]), x["S0"][0, 0], sel(gO), gS[0, 0], gate_mode, scale,
                                  sel(x["w"]))
    o2, S2, g2 = bwd.chunk_bwd_head(*args, x["S0"][0, 0], sel(gO), gS[0, 0], gate_mode, scale, sel(x["w"]), chunk,
                                    theta=sel(x["theta"]))
    assert np.max(np.abs(o2 - o1)) < 1e-10 * np.max(np.abs(o1)) and np.max(np.abs(S2 - S1)) < 1e-10 * np.max(np.abs(S1))
    for n in ("q", "k", "v", "g", "beta", "S0") + (("w",) if untied else ()) + (("theta",) if rotation else ()):
        assert np.max(np.abs(g2[n] - g1[n])) < 1e-9 * max(np.max(np.abs(g1[n])), 1e-12), n
