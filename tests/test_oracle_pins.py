"""Pins for the fp64 oracle: brute force, the pages' chunk algebra, invariants, closed forms.

Nothing here retypes the oracle's loop.  Each check computes the same quantity
another way (explicit products of transition matrices, the SFDA constructive
chunk-WY product, closed forms of special cases) or checks a property the
mathematics fixes, so that a dropped term, a wrong sign, a swapped index or a
transposed operand in the oracle fails at least one of them.
"""
import json
import os

import numpy as np
import pytest

import oracle
from oracle import chunk_wy

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _rand_problem(rng, B, T, H, dk, dv, rotation=False, s0=True, unit_k=True):
    q = rng.standard_normal((B, T, H, dk))
    k = rng.standard_normal((B, T, H, dk))
    if unit_k:
        k /= np.linalg.norm(k, axis=-1, keepdims=True)
        q /= np.linalg.norm(q, axis=-1, keepdims=True)
    v = rng.standard_normal((B, T, H, dv))
    ng = dk // 2 if rotation else dk
    a = rng.standard_normal((B, T, H, ng))
    beta = 1.0 / (1.0 + np.exp(-rng.standard_normal((B, T, H))))
    theta = rng.uniform(-np.pi, np.pi, (B, T, H, dk // 2)) if rotation else None
    S0 = rng.standard_normal((B, H, dv, dk)) * 0.5 if s0 else None
    return q, k, v, a, beta, theta, S0


def _decay_by_complex(a_t, theta_t, dk):
    """D_t built independently: alpha = sigmoid(-a) (= exp(-softplus(a))); in
    rotation mode each key pair of a row vector is a complex number multiplied by
    alpha e^{i theta}.  Rows of D are the images of the basis row vectors."""
    alpha = 1.0 / (1.0 + np.exp(a_t))
    if theta_t is None:
        return np.diag(alpha)
    D = np.zeros((dk, dk))
    for j in range(dk // 2):
        w = alpha[j] * np.exp(1j * theta_t[j])
        for src, z in ((2 * j, 1.0 + 0j), (2 * j + 1, 1j)):
            img = z * w
            D[src, 2 * j] = img.real
            D[src, 2 * j + 1] = img.imag
    return D


def _brute_head(q, k, v, a, beta, theta, S0, scale, w=None):
    """S_t = S_0 prod_{s<=t} M_s + sum_{i<=t} w_i v_i k_i^T prod_{i<s<=t} M_s with
    M_s = D_s (I - beta_s k_s k_s^T), every product formed explicitly (w = beta: the
    tied delta rule; otherwise beta erases and w writes)."""
    w = beta if w is None else w
    T, dk = q.shape
    dv = v.shape[1]
    M = []
    for t in range(T):
        D = _decay_by_complex(a[t], None if theta is None else theta[t], dk)
        M.append(D @ (np.eye(dk) - beta[t] * np.outer(k[t], k[t])))

    def prod(lo, hi):
        P = np.eye(dk)
        for s in range(lo, hi):
            P = P @ M[s]
        return P

    S0 = np.zeros((dv, dk)) if S0 is None else S0
    o = np.zeros((T, dv))
    S_t = None
    for t in range(T):
        S_t = S0 @ prod(0, t + 1)
        for i in range(t + 1):
            S_t = S_t + w[i] * np.outer(v[i], k[i]) @ prod(i + 1, t + 1)
        o[t] = S_t @ (scale * q[t])
    return o, S_t


def _rel(a, b):
    return np.max(np.abs(a - b)) / max(np.max(np.abs(b)), 1e-300)


@pytest.mark.parametrize("rotation", [False, True])
def test_oracle_matches_brute_force_products(rotation):
    rng = np.random.default_rng(11 + rotation)
    B, T, H, dk, dv = 2, 13, 2, 8, 6
    q, k, v, a, beta, theta, S0 = _rand_problem(rng, B, T, H, dk, dv, rotation)
    o, S_T = oracle.gdr_fwd(q, k, v, a, beta, theta, S0, oracle.GATE_NEG_SOFTPLUS, scale=0.7)
    for b in range(B):
        for h in range(H):
            ob, Sb = _brute_head(q[b, :, h], k[b, :, h], v[b, :, h], a[b, :, h], beta[b, :, h],
                                 None if theta is None else theta[b, :, h], S0[b, h], 0.7)
            assert _rel(o[b, :, h], ob) < 1e-12
            assert _rel(S_T[b, h], Sb) < 1e-12


def test_brute_force_pin_catches_planted_mistakes():
    """The brute-force pin is sharp enough to see plausible mistakes: an erase
    applied before the decay, a transposed decay block, and a readout with the
    pre-update state all move the result far above the tolerance."""
    rng = np.random.default_rng(5)
    T, dk, dv = 9, 6, 4
    q, k, v, a, beta, theta, S0 = _rand_problem(rng, 1, T, 1, dk, dv, rotation=True)
    q, k, v, a, beta, theta, S0 = (q[0, :, 0], k[0, :, 0], v[0, :, 0], a[0, :, 0],
                                  beta[0, :, 0], theta[0, :, 0], S0[0, 0])
    o_ref, S_ref = _brute_head(q, k, v, a, beta, theta, S0, 1.0)

    def run(variant):
        S = S0.copy()
        o = np.zeros((T, dv))
        for t in range(T):
            D = _decay_by_complex(a[t], theta[t], dk)
            if variant == "transposed_block":
                D = D.T
            if variant == "erase_first":
                S = S @ (np.eye(dk) - beta[t] * np.outer(k[t], k[t])) @ D
                S = S + beta[t] * np.outer(v[t], k[t])
            else:
                X = S @ D
                e = beta[t] * (v[t] - X @ k[t])
                S_new = X + np.outer(e, k[t])
                if variant == "pre_update_readout":
                    o[t] = S @ q[t]
                    S = S_new
                    continue
                S = S_new
            o[t] = S @ q[t]
        return o, S

    o_ok, S_ok = run("none")
    assert _rel(o_ok, o_ref) < 1e-12 and _rel(S_ok, S_ref) < 1e-12
    for variant in ("transposed_block", "erase_first", "pre_update_readout"):
        o_bad, _ = run(variant)
        assert _rel(o_bad, o_ref) > 1e-3, variant


@pytest.mark.parametrize("rotation", [False, True])
def test_sfda_constructive_chunk_wy_matches_oracle(rotation):
    """Constructive chunk-WY product + affine chunk transfer == token recurrence,
    within the page's reported verification residuals."""
    bounds = json.load(open(os.path.join(GOLDEN, "verification_residuals.json")))
    rng = np.random.default_rng(21 + rotation)
    T, dk, dv, C = 23, 8, 5, 6                       # ragged tail: 23 = 3*6 + 5
    q, k, v, a, beta, theta, S0 = _rand_problem(rng, 1, T, 1, dk, dv, rotation)
    o_ref, S_ref = oracle.gdr_fwd(q, k, v, a, beta, theta, S0, oracle.GATE_NEG_SOFTPLUS, 0.9)
    sl = lambda x: None if x is None else x[0, :, 0]
    o, S, transfers = chunk_wy.sfda_chunk_wy(sl(q), sl(k), sl(v), sl(a), sl(beta), sl(theta),
                                             S0[0, 0], chunk=C,
                                             gate_mode=chunk_wy.GATE_NEG_SOFTPLUS, scale=0.9)
    assert _rel(o, o_ref[0, :, 0]) < bounds["residual_max"]
    assert _rel(S, S_ref[0, 0]) < bounds["residual_max"]


def test_chunk_transition_rank_bounded_by_chunk():
    """Inside a chunk the correction P_C - Gamma_C has rank <= C (it resets at the
    chunk boundary), checked on the explicitly multiplied transition matrices."""
    rng = np.random.default_rng(3)
    dk, C = 24, 5
    q, k, v, a, beta, theta, _ = _rand_problem(rng, 1, C, 1, dk, 2, rotation=True, s0=False)
    P = np.eye(dk)
    Gam = np.eye(dk)
    for t in range(C):
        D = _decay_by_complex(a[0, t, 0], theta[0, t, 0], dk)
        Lam = D.T                                     # page orientation acts from the left
        A_t = Lam - beta[0, t, 0] * np.outer(k[0, t, 0], Lam.T @ k[0, t, 0])
        P = A_t @ P
        Gam = Lam @ Gam
    sv = np.linalg.svd(P - Gam, compute_uv=False)
    assert np.sum(sv > 1e-10 * sv[0]) == C
    # and the constructive form reproduces the explicit product
    _, _, transfers = chunk_wy.sfda_chunk_wy(q[0, :, 0], k[0, :, 0], v[0, :, 0], a[0, :, 0],
                                             beta[0, :, 0], theta[0, :, 0], None, chunk=C,
                                             gate_mode=chunk_wy.GATE_NEG_SOFTPLUS)
    P_C, Gam_C, _ = transfers[0]
    assert np.max(np.abs(P_C - P)) < 1e-12 and np.max(np.abs(Gam_C - Gam)) < 1e-12


@pytest.mark.parametrize("rotation", [False, True])
def test_ut_transform_chunk_matches_oracle(rotation):
    """The UT-transform chunk solver the kernels evaluate == token recurrence."""
    rng = np.random.default_rng(31 + rotation)
    T, dk, dv, C = 29, 8, 6, 8
    q, k, v, a, beta, theta, S0 = _rand_problem(rng, 1, T, 1, dk, dv, rotation)
    o_ref, S_ref = oracle.gdr_fwd(q, k, v, a, beta, theta, S0, oracle.GATE_NEG_SOFTPLUS, 1.3)
    sl = lambda x: None if x is None else x[0, :, 0]
    o, S = chunk_wy.ut_chunk(sl(q), sl(k), sl(v), sl(a), sl(beta), sl(theta), S0[0, 0], chunk=C,
                             gate_mode=chunk_wy.GATE_NEG_SOFTPLUS, scale=1.3)
    assert _rel(o, o_ref[0, :, 0]) < 1e-11
    assert _rel(S, S_ref[0, 0]) < 1e-11


def test_zero_phase_reduces_to_real_decay():
    """Tied SFDA recovers KDA at phase zero: rotation mode with theta = 0 equals
    real mode with each pair's gate repeated on both of its key dims."""
    rng = np.random.default_rng(41)
    B, T, H, dk, dv = 1, 17, 2, 8, 4
    q, k, v, a, beta, theta, S0 = _rand_problem(rng, B, T, H, dk, dv, rotation=True)
    o_rot, S_rot = oracle.gdr_fwd(q, k, v, a, beta, np.zeros_like(theta), S0,
                                  oracle.GATE_NEG_SOFTPLUS)
    o_real, S_real = oracle.gdr_fwd(q, k, v, np.repeat(a, 2, axis=-1), beta, None, S0,
                                    oracle.GATE_NEG_SOFTPLUS)
    assert _rel(o_rot, o_real) < 1e-14 and _rel(S_rot, S_real) < 1e-14


def test_no_decay_no_write_keeps_state():
    rng = np.random.default_rng(51)
    B, T, H, dk, dv = 1, 11, 2, 8, 5
    q, k, v, _, _, _, S0 = _rand_problem(rng, B, T, H, dk, dv)
    g = np.zeros((B, T, H, dk))
    beta = np.zeros((B, T, H))
    o, S_T = oracle.gdr_fwd(q, k, v, g, beta, None, S0, oracle.GATE_LOGDECAY)
    assert np.array_equal(S_T, S0)
    expect = np.einsum("bhij,bthj->bthi", S0, q)
    assert _rel(o, expect) < 1e-14


def test_full_write_stores_value_along_unit_key():
    """beta = 1 and |k| = 1: (I - k k^T) k = 0, so S_t k_t = v_t for any decay and
    phase.  With q_t = k_t the readout returns v_t."""
    rng = np.random.default_rng(61)
    for rotation in (False, True):
        q, k, v, a, beta, theta, S0 = _rand_problem(rng, 2, 15, 2, 8, 6, rotation)
        o, _ = oracle.gdr_fwd(k, k, v, a, np.ones_like(beta), theta, S0, oracle.GATE_NEG_SOFTPLUS)
        assert np.max(np.abs(o - v)) < 1e-13


def test_pure_decay_closed_form():
    """beta = 0: S_T = S_0 diag(prod_t sigmoid(-a_t)) (real mode) and, with phase,
    each key pair is multiplied by prod(alpha) * e^{i sum(theta)}."""
    rng = np.random.default_rng(71)
    B, T, H, dk, dv = 1, 20, 2, 8, 3
    q, k, v, a, beta, theta, S0 = _rand_problem(rng, B, T, H, dk, dv, rotation=True)
    a = a * 10.0                                     # include strongly saturated gates
    zb = np.zeros_like(beta)
    _, S_T = oracle.gdr_fwd(q, k, v, np.repeat(a, 2, -1), zb, None, S0, oracle.GATE_NEG_SOFTPLUS)
    decay = np.prod(1.0 / (1.0 + np.exp(np.repeat(a, 2, -1))), axis=1)      # [B,H,dk]
    assert _rel(S_T, S0 * decay[:, :, None, :]) < 1e-13
    _, S_rot = oracle.gdr_fwd(q, k, v, a, zb, theta, S0, oracle.GATE_NEG_SOFTPLUS)
    w = np.prod(1.0 / (1.0 + np.exp(a)), axis=1) * np.exp(1j * np.sum(theta, axis=1))
    z0 = S0[..., 0::2] + 1j * S0[..., 1::2]
    z = z0 * w[:, :, None, :]
    expect = np.empty_like(S0)
    expect[..., 0::2], expect[..., 1::2] = z.real, z.imag
    assert _rel(S_rot, expect) < 1e-12


def test_gate_activation_extremes():
    """-softplus stays finite and exact for large |a|: a = +40 decays by e^{-40}
    per token, a = -40 keeps the state (alpha = 1 - e^{-40})."""
    dk, dv, T = 4, 2, 3
    S0 = np.ones((1, 1, dv, dk))
    z = np.zeros((1, T, 1, dk))
    for aval in (40.0, -40.0, 0.0, 700.0):
        a = np.full((1, T, 1, dk), aval)
        _, S_T = oracle.gdr_fwd(z, z, np.zeros((1, T, 1, dv)), a, np.zeros((1, T, 1)), None, S0,
                                oracle.GATE_NEG_SOFTPLUS)
        expect = (1.0 / (1.0 + np.exp(aval))) ** T if aval < 700 else 0.0
        assert np.all(np.isfinite(S_T))
        assert abs(S_T[0, 0, 0, 0] - expect) <= 1e-15 + 1e-13 * expect


def test_phase_only_counter_is_periodic():
    """Phase-only memory (beta = 0, g = 0, theta = 2 pi / 5) is a mod-5 counter: the
    state returns to itself every 5 tokens, exactly over the lengths the page
    reports (27 to 213)."""
    gold = json.load(open(os.path.join(GOLDEN, "counter_mod5.json")))
    period = gold["period"]
    lo, hi = gold["lengths"]
    rng = np.random.default_rng(81)
    dk, dv = 4, 3
    S0 = rng.standard_normal((1, 1, dv, dk))
    for T in (lo, lo + 1, hi - 3, hi):
        z = np.zeros((1, T, 1, dk))
        theta = np.full((1, T, 1, dk // 2), 2.0 * np.pi / period)
        _, S_T = oracle.gdr_fwd(z, z, np.zeros((1, T, 1, dv)), np.zeros((1, T, 1, dk // 2)),
                                np.zeros((1, T, 1)), theta, S0, oracle.GATE_LOGDECAY)
        _, S_r = oracle.gdr_fwd(z[:, :T % period], z[:, :T % period],
                                np.zeros((1, T % period, 1, dv)),
                                np.zeros((1, T % period, 1, dk // 2)), np.zeros((1, T % period, 1)),
                                theta[:, :T % period], S0, oracle.GATE_LOGDECAY)
        assert np.max(np.abs(S_T - S_r)) < gold["residual_bound"]


def test_state_norm_contracts():
    """With no write (v = 0), a unit key and beta in [0,1], ||S_t||_F never grows:
    ||I - beta k k^T||_2 <= 1, rotations are orthogonal and decays are <= 1."""
    rng = np.random.default_rng(91)
    for rotation in (False, True):
        T, dk, dv = 40, 8, 6
        q, k, v, a, beta, theta, S0 = _rand_problem(rng, 1, T, 1, dk, dv, rotation)
        norms = [np.linalg.norm(S0)]
        S = S0
        for t in range(T):
            sl = slice(t, t + 1)
            _, S = oracle.gdr_fwd(q[:, sl], k[:, sl], np.zeros((1, 1, 1, dv)), a[:, sl],
                                  beta[:, sl], None if theta is None else theta[:, sl], S,
                                  oracle.GATE_NEG_SOFTPLUS)
            norms.append(np.linalg.norm(S))
        norms = np.array(norms)
        assert np.all(np.diff(norms) <= 1e-14 * norms[:-1])


def test_output_is_linear_in_initial_state_and_values():
    """o and S_T are linear in (S_0, v) jointly for fixed q, k, g, beta, theta."""
    rng = np.random.default_rng(101)
    q, k, v1, a, beta, theta, S1 = _rand_problem(rng, 1, 19, 2, 8, 5, rotation=True)
    _, _, v2, _, _, _, S2 = _rand_problem(rng, 1, 19, 2, 8, 5, rotation=True)
    f = lambda v, S: oracle.gdr_fwd(q, k, v, a, beta, theta, S, oracle.GATE_NEG_SOFTPLUS)
    o1, T1 = f(v1, S1)
    o2, T2 = f(v2, S2)
    o3, T3 = f(2.0 * v1 - 0.5 * v2, 2.0 * S1 - 0.5 * S2)
    assert _rel(o3, 2.0 * o1 - 0.5 * o2) < 1e-12
    assert _rel(T3, 2.0 * T1 - 0.5 * T2) < 1e-12


@pytest.mark.parametrize("t0", [1, 7, 16, 31])
def test_split_sequence_resumes_from_state(t0):
    rng = np.random.default_rng(111)
    q, k, v, a, beta, theta, S0 = _rand_problem(rng, 2, 32, 2, 8, 4, rotation=False)
    o, S_T = oracle.gdr_fwd(q, k, v, a, beta, None, S0, oracle.GATE_NEG_SOFTPLUS)
    oa, Sa = oracle.gdr_fwd(q[:, :t0], k[:, :t0], v[:, :t0], a[:, :t0], beta[:, :t0], None, S0,
                            oracle.GATE_NEG_SOFTPLUS)
    ob, Sb = oracle.gdr_fwd(q[:, t0:], k[:, t0:], v[:, t0:], a[:, t0:], beta[:, t0:], None, Sa,
                            oracle.GATE_NEG_SOFTPLUS)
    assert np.array_equal(np.concatenate([oa, ob], axis=1), o)
    assert np.array_equal(Sb, S_T)


def test_single_token_closed_form_and_orientation():
    """T = 1, S_0 = 0: S_1 = beta v k^T and o_1 = beta (k.q) v (the readout uses the
    post-update state).  With S_0 != 0, beta = 0, g = 0: o = S_0 q (S is dv x dk)."""
    rng = np.random.default_rng(121)
    q, k, v, a, beta, _, S0 = _rand_problem(rng, 1, 1, 1, 6, 3)
    o, S1 = oracle.gdr_fwd(q, k, v, a, beta, None, None, oracle.GATE_NEG_SOFTPLUS)
    bq = beta[0, 0, 0]
    assert _rel(S1[0, 0], bq * np.outer(v[0, 0, 0], k[0, 0, 0])) < 1e-15
    assert _rel(o[0, 0, 0], bq * np.dot(k[0, 0, 0], q[0, 0, 0]) * v[0, 0, 0]) < 1e-14
    o, _ = oracle.gdr_fwd(q, k, v, np.zeros_like(a), np.zeros_like(beta), None, S0,
                          oracle.GATE_LOGDECAY)
    assert _rel(o[0, 0, 0], S0[0, 0] @ q[0, 0, 0]) < 1e-15
    assert not np.allclose(o[0, 0, 0], S0[0, 0].T[:3, :3] @ q[0, 0, 0][:3])


@pytest.mark.parametrize("rotation", [False, True])
def test_decode_steps_equal_forward(rotation):
    rng = np.random.default_rng(131 + rotation)
    T = 6
    q, k, v, a, beta, theta, S0 = _rand_problem(rng, 3, T, 2, 8, 4, rotation)
    o, S_T = oracle.gdr_fwd(q, k, v, a, beta, theta, S0, oracle.GATE_NEG_SOFTPLUS, 0.8)
    S = S0
    for t in range(T):
        od, S = oracle.gdr_decode_step(q[:, t], k[:, t], v[:, t], a[:, t], beta[:, t], S,
                                       None if theta is None else theta[:, t],
                                       oracle.GATE_NEG_SOFTPLUS, 0.8)
        assert np.array_equal(od, o[:, t])
    assert np.array_equal(S, S_T)


# ---- separate erase and write strengths ("CARVE" page, sections 2.1-2.2) ----------------

def _write_gate(rng, shape):
    return 1.0 / (1.0 + np.exp(-rng.standard_normal(shape)))


@pytest.mark.parametrize("rotation", [False, True])
def test_untied_oracle_matches_brute_force_products(rotation):
    rng = np.random.default_rng(71 + rotation)
    B, T, H, dk, dv = 2, 11, 2, 8, 6
    q, k, v, a, beta, theta, S0 = _rand_problem(rng, B, T, H, dk, dv, rotation)
    w = _write_gate(rng, (B, T, H))
    o, S_T = oracle.gdr_fwd(q, k, v, a, beta, theta, S0, oracle.GATE_NEG_SOFTPLUS, scale=0.9, w=w)
    for b in range(B):
        for h in range(H):
            ob, Sb = _brute_head(q[b, :, h], k[b, :, h], v[b, :, h], a[b, :, h], beta[b, :, h],
                                 None if theta is None else theta[b, :, h], S0[b, h], 0.9, w=w[b, :, h])
            assert _rel(o[b, :, h], ob) < 1e-12
            assert _rel(S_T[b, h], Sb) < 1e-12
    # the pin separates the two gates: exchanging them moves the result far
    o_x, _ = _brute_head(q[0, :, 0], k[0, :, 0], v[0, :, 0], a[0, :, 0], w[0, :, 0],
                         None if theta is None else theta[0, :, 0], S0[0, 0], 0.9, w=beta[0, :, 0])
    assert _rel(o_x, o[0, :, 0]) > 1e-3


def test_untied_with_write_equal_to_erase_is_the_delta_rule():
    rng = np.random.default_rng(72)
    q, k, v, a, beta, theta, S0 = _rand_problem(rng, 1, 20, 2, 8, 5)
    o1, S1 = oracle.gdr_fwd(q, k, v, a, beta, theta, S0, oracle.GATE_NEG_SOFTPLUS)
    o2, S2 = oracle.gdr_fwd(q, k, v, a, beta, theta, S0, oracle.GATE_NEG_SOFTPLUS, w=beta.copy())
    assert np.array_equal(o1, o2) and np.array_equal(S1, S2)


def test_write_only_without_decay_is_a_running_sum():
    """beta = 0, g = 0: nothing is erased or decayed, so S_t = S_0 + sum_{i<=t} w_i v_i k_i^T
    and o_t = S_t q_t, written out as cumulative sums."""
    rng = np.random.default_rng(73)
    q, k, v, a, beta, theta, S0 = _rand_problem(rng, 1, 17, 1, 6, 4, unit_k=False)
    w = rng.standard_normal((1, 17, 1))
    zero = np.zeros_like(beta)
    o, S_T = oracle.gdr_fwd(q, k, v, np.zeros_like(a), zero, None, S0, oracle.GATE_LOGDECAY, w=w)
    terms = w[0, :, 0, None, None] * v[0, :, 0, :, None] * k[0, :, 0, None, :]
    S_run = S0[0, 0][None] + np.cumsum(terms, axis=0)
    assert _rel(S_T[0, 0], S_run[-1]) < 1e-13
    assert _rel(o[0, :, 0], np.einsum("tij,tj->ti", S_run, q[0, :, 0])) < 1e-13


def test_erase_only_annihilates_the_key():
    """w = 0, beta = 1, unit keys, no decay: each step projects the state off k_t, so
    S_t k_t = 0 and nothing of v is written."""
    rng = np.random.default_rng(74)
    q, k, v, a, beta, theta, S0 = _rand_problem(rng, 1, 6, 1, 8, 5)
    ones, zero = np.ones_like(beta), np.zeros_like(beta)
    for t in range(1, 7):
        _, S = oracle.gdr_fwd(q[:, :t], k[:, :t], v[:, :t], np.zeros_like(a[:, :t]), ones[:, :t], None, S0,
                              oracle.GATE_LOGDECAY, w=zero[:, :t])
        assert np.max(np.abs(S[0, 0] @ k[0, t - 1, 0])) < 1e-13


def test_untied_decode_steps_equal_forward():
    rng = np.random.default_rng(75)
    q, k, v, a, beta, theta, S0 = _rand_problem(rng, 1, 9, 3, 8, 6, rotation=True)
    w = _write_gate(rng, (1, 9, 3))
    o_f, S_f = oracle.gdr_fwd(q, k, v, a, beta, theta, S0, oracle.GATE_NEG_SOFTPLUS, w=w)
    S = S0.copy()
    for t in range(9):
        o_t, S = oracle.gdr_decode_step(q[:, t], k[:, t], v[:, t], a[:, t], beta[:, t], S, theta[:, t],
                                        oracle.GATE_NEG_SOFTPLUS, w=w[:, t])
        assert _rel(o_t, o_f[:, t]) < 1e-12
    assert _rel(S, S_f) < 1e-12


# ---- fused L2 normalisation of q and k (NEXT-4 prologue) ---------------------------------

def test_l2norm_prologue_makes_the_layer_blind_to_key_and_query_scale():
    """With the prologue on, rescaling each token's q and k by arbitrary positive factors
    changes nothing (up to the 1e-6 epsilon); with it off, the same rescaling changes the
    result a lot."""
    rng = np.random.default_rng(81)
    q, k, v, a, beta, theta, S0 = _rand_problem(rng, 1, 23, 2, 8, 5, rotation=True)
    fq = np.exp(rng.uniform(0, 2, q.shape[:-1] + (1,)))       # norms >= 1: epsilon below 1e-6
    fk = np.exp(rng.uniform(0, 2, k.shape[:-1] + (1,)))
    o1, S1 = oracle.gdr_fwd(q, k, v, a, beta, theta, S0, oracle.GATE_NEG_SOFTPLUS, qk_l2norm=True)
    o2, S2 = oracle.gdr_fwd(q * fq, k * fk, v, a, beta, theta, S0, oracle.GATE_NEG_SOFTPLUS, qk_l2norm=True)
    assert _rel(o2, o1) < 1e-5 and _rel(S2, S1) < 1e-5
    o3, _ = oracle.gdr_fwd(q * fq, k * fk, v, a, beta, theta, S0, oracle.GATE_NEG_SOFTPLUS)
    assert _rel(o3, o1) > 1e-2


def test_l2norm_prologue_on_unit_inputs_changes_only_by_epsilon():
    rng = np.random.default_rng(82)
    q, k, v, a, beta, theta, S0 = _rand_problem(rng, 2, 15, 2, 8, 6)       # unit q, k
    o1, S1 = oracle.gdr_fwd(q, k, v, a, beta, theta, S0, oracle.GATE_NEG_SOFTPLUS)
    o2, S2 = oracle.gdr_fwd(q, k, v, a, beta, theta, S0, oracle.GATE_NEG_SOFTPLUS, qk_l2norm=True)
    assert _rel(o2, o1) < 1e-5 and _rel(S2, S1) < 1e-5


def test_l2norm_prologue_keeps_zero_vectors_zero_and_decode_agrees():
    rng = np.random.default_rng(83)
    q, k, v, a, beta, theta, S0 = _rand_problem(rng, 1, 7, 3, 8, 4, unit_k=False)
    q[0, 3] = 0.0                                   # a zero query reads nothing
    o, S_f = oracle.gdr_fwd(q, k, v, a, beta, None, S0, oracle.GATE_NEG_SOFTPLUS, qk_l2norm=True)
    assert np.all(o[0, 3] == 0.0)
    S = S0.copy()
    for t in range(7):
        o_t, S = oracle.gdr_decode_step(q[:, t], k[:, t], v[:, t], a[:, t], beta[:, t], S, None,
                                        oracle.GATE_NEG_SOFTPLUS, qk_l2norm=True)
        assert _rel(o_t + 1e-300, o[:, t] + 1e-300) < 1e-12 or np.all(o[:, t] == o_t)
    assert _rel(S, S_f) < 1e-12


def _l2norm_epsilon_pin_holds(normalise):
    """The stated convention puts the 1e-6 inside the square root: for x = c u with a unit u,
    the result is u c / sqrt(c^2 + 1e-6).  Choosing c^2 as a multiple of 1e-6 makes that
    norm a known number: c^2 = 3e-6 gives sqrt(3)/2, c^2 = 1e-6 gives 1/sqrt(2), c^2 = 8e-6
    gives sqrt(8)/3.  The direction of x is kept."""
    rng = np.random.default_rng(91)
    for mult, norm in ((3.0, np.sqrt(3.0) / 2.0), (1.0, 1.0 / np.sqrt(2.0)), (8.0, np.sqrt(8.0) / 3.0)):
        u = rng.normal(size=(4, 16))
        u /= np.linalg.norm(u, axis=-1, keepdims=True)
        y = np.asarray(normalise(u * np.sqrt(mult * 1e-6)), dtype=np.float64)
        if not np.allclose(np.linalg.norm(y, axis=-1), norm, rtol=1e-9, atol=0):
            return False
        if not np.allclose(y / np.linalg.norm(y, axis=-1, keepdims=True), u, rtol=1e-9, atol=1e-12):
            return False
    return True


def test_l2norm_epsilon_sits_inside_the_root_with_value_1e_6():
    assert _l2norm_epsilon_pin_holds(oracle.l2_normalise)


def test_l2norm_epsilon_pin_catches_planted_mistakes():
    planted = {
        "epsilon outside the root": lambda x: x / (np.sqrt(np.sum(x * x, -1, keepdims=True)) + 1e-6),
        "epsilon 1e-12": lambda x: x / np.sqrt(np.sum(x * x, -1, keepdims=True) + 1e-12),
        "no epsilon": lambda x: x / np.sqrt(np.sum(x * x, -1, keepdims=True)),
    }
    for name, f in planted.items():
        assert not _l2norm_epsilon_pin_holds(f), name


def test_l2norm_epsilon_reaches_the_forward():
    """One token from the zero state, q = k = c u with c^2 = 3e-6: S_1 = beta v khat^T and
    o_1 = beta v (khat . qhat) = beta v c^2 / (c^2 + 1e-6) = 0.75 beta v, whatever the gate."""
    rng = np.random.default_rng(92)
    H, d = 3, 8
    u = rng.normal(size=(1, 1, H, d))
    u /= np.linalg.norm(u, axis=-1, keepdims=True)
    q = k = u * np.sqrt(3e-6)
    v = rng.normal(size=(1, 1, H, 5))
    a = rng.normal(size=(1, 1, H, d))
    beta = rng.uniform(0.2, 0.9, size=(1, 1, H))
    o, _ = oracle.gdr_fwd(q, k, v, a, beta, None, None, oracle.GATE_NEG_SOFTPLUS, qk_l2norm=True)
    assert np.allclose(o, 0.75 * beta[..., None] * v, rtol=1e-10, atol=0)


# ---- chunk means of the output (the content signal of CARVE's content-aware erase) -------

@pytest.mark.parametrize("T,chunk", [(150, 64), (64, 64), (37, 16), (1, 64)])
def test_chunk_means_of_a_ramp_are_the_chunk_midpoints(T, chunk):
    """o_t = t (every head and value row): the mean over tokens t0 .. t1-1 of a chunk is the
    midpoint (t0 + t1 - 1) / 2 of an arithmetic series, the last chunk cut at T."""
    o = np.broadcast_to(np.arange(T, dtype=np.float64)[None, :, None, None], (2, T, 3, 4)).copy()
    m = oracle.chunk_means(o, chunk)
    nc = -(-T // chunk)
    assert m.shape == (2, nc, 3, 4)
    for c in range(nc):
        t0, t1 = c * chunk, min((c + 1) * chunk, T)
        assert np.all(m[:, c] == (t0 + t1 - 1) / 2.0)


def test_chunk_means_of_piecewise_constant_outputs_and_total_mass():
    """o constant within each chunk returns that constant; and sum_c L_c m_c is the sum of
    o over the whole sequence, for any o."""
    rng = np.random.default_rng(91)
    T, chunk = 200, 64
    levels = rng.standard_normal((1, 4, 2, 5))
    o = np.repeat(levels, chunk, axis=1)[:, :T]
    assert _rel(oracle.chunk_means(o, chunk), levels) < 1e-14
    o = rng.standard_normal((2, T, 3, 5))
    m = oracle.chunk_means(o, chunk)
    L = np.array([64, 64, 64, 8], dtype=np.float64)
    assert _rel(np.einsum("bchd,c->bhd", m, L), o.sum(axis=1)) < 1e-13


def test_chunk_means_of_a_full_write_are_the_value_means():
    """beta = 1, unit keys, q_t = k_t: the readout returns v_t (S_t k_t = v_t), so the
    chunk means of the recurrence's output are the chunk means of v, a closed form that
    does not pass through the recurrence."""
    rng = np.random.default_rng(92)
    q, k, v, a, beta, theta, S0 = _rand_problem(rng, 1, 70, 2, 8, 6, rotation=True)
    o, _ = oracle.gdr_fwd(k, k, v, a, np.ones_like(beta), theta, S0, oracle.GATE_NEG_SOFTPLUS)
    m = oracle.chunk_means(o, 64)
    assert _rel(m[:, 0], v[:, :64].mean(axis=1)) < 1e-12
    assert _rel(m[:, 1], v[:, 64:].mean(axis=1)) < 1e-12


def test_chunk_mean_pins_catch_planted_mistakes():
    """The ramp closed form sees plausible mistakes in a chunk mean: a short last chunk divided
    by the full chunk length, chunk boundaries off by one token, and the mean taken over the
    wrong axis."""
    T, chunk = 150, 64
    # o[b, t, h, j] = t (j + 1): value rows carry different ramps, so the axis matters
    o = np.arange(T, dtype=np.float64)[None, :, None, None] * np.arange(1, 4)[None, None, None, :]
    o = np.broadcast_to(o, (1, T, 2, 3)).copy()
    nc = -(-T // chunk)

    def expect(c):
        t0, t1 = c * chunk, min((c + 1) * chunk, T)
        return o[:, t0:t1].sum(axis=1) / (t1 - t0)

    def planted(variant):
        m = np.zeros((1, nc, 2, 3))
        for c in range(nc):
            t0, t1 = c * chunk, min((c + 1) * chunk, T)
            if variant == "full_divisor":
                m[:, c] = o[:, t0:t1].sum(axis=1) / chunk
            elif variant == "shifted":
                m[:, c] = o[:, t0 + 1:t1 + 1].mean(axis=1)
            elif variant == "wrong_axis":
                m[:, c] = o[:, t0:t1].mean(axis=-1, keepdims=True).mean(axis=1)
        return m

    m = oracle.chunk_means(o, chunk)
    for c in range(nc):
        assert _rel(m[:, c], expect(c)) < 1e-15
        assert np.all(m[0, c, 0, 0] == (c * chunk + min((c + 1) * chunk, T) - 1) / 2.0)
    for variant in ("full_divisor", "shifted", "wrong_axis"):
        bad = planted(variant)
        assert max(_rel(bad[:, c], expect(c)) for c in range(nc)) > 1e-3, variant


# ---- sequence-parallel form: segments joined by the affine state transfer (NEXT-3) ---------

@pytest.mark.parametrize("T,segment,rotation,untied", [(200, 64, False, False), (130, 50, True, True),
                                                       (97, 256, True, False), (64, 1, False, True)])
def test_segment_scan_equals_the_token_recurrence(T, segment, rotation, untied):
    """Segments computed independently (from the zero state and from the identity), joined by
    a sequential scan of S_{s+1} = S_s A_s + B_s and an output correction S_s A_{s,t} q_t,
    reproduce the token recurrence: segment lengths that divide T, that do not, a single
    segment and one-token segments."""
    rng = np.random.default_rng(600 + T)
    q, k, v, a, beta, theta, S0 = _rand_problem(rng, 1, T, 1, 8, 6, rotation)
    w = _write_gate(rng, (1, T, 1)) if untied else None
    sel = lambda x: None if x is None else x[0, :, 0]
    o_ref, S_ref = oracle.gdr_fwd(q, k, v, a, beta, theta, S0, oracle.GATE_NEG_SOFTPLUS, w=w)
    o, S = oracle.segment_scan(sel(q), sel(k), sel(v), sel(a), sel(beta), sel(theta), S0[0, 0], segment,
                               oracle.GATE_NEG_SOFTPLUS, w=sel(w))
    assert _rel(o, o_ref[0, :, 0]) < 1e-11 and _rel(S, S_ref[0, 0]) < 1e-11
