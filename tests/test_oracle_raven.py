"""Pins of the Raven slot-memory oracle (oracle/raven.py) against what the page and the
mathematics fix: the router's top-K selection by brute force, the special case that section 2.1
names (a one-hot router with an emptying decay is sliding-window attention, written here as
plain attention over the window), frozen slots, the dense equal router as an exponential moving
average in closed form, the chunked restatement against the token loop, and planted mistakes
that these pins must catch."""
import numpy as np
import pytest

from oracle import raven as R


def _rand(rng, B, T, H, dk, dv, M):
    q = rng.standard_normal((B, T, H, dk))
    k = rng.standard_normal((B, T, H, dk))
    v = rng.standard_normal((B, T, H, dv))
    z = rng.standard_normal((B, T, H, M)).astype(np.float32)
    g = rng.standard_normal((B, T, H))
    return q, k, v, z, g


def test_router_matches_brute_force_selection():
    """Top K by a plain sort of (-logit, slot) pairs, ties to the lower slot; the kept sigmoid
    scores normalised to one."""
    rng = np.random.default_rng(500)
    z = rng.integers(-3, 4, size=(40, 9)).astype(np.float32)        # many ties
    for K in (1, 3, 9):
        idx, r = R.route(z, K)
        for n in range(z.shape[0]):
            order = sorted(range(9), key=lambda i: (-float(z[n, i]), i))[:K]
            assert list(idx[n]) == order
            m = np.array([1.0 / (1.0 + np.exp(-float(z[n, i]))) for i in order])
            want = np.zeros(9)
            want[order] = m / m.sum()
            assert np.allclose(r[n], want, rtol=0, atol=1e-15)
            assert abs(r[n].sum() - 1.0) < 1e-15


def _swa(q, k, v, S0k, S0v, M, scale):
    """Attention over the last M tokens' keys and values; slots not yet written hold S0's rows
    (slot j holds the latest token s <= t with s mod M == j)."""
    T = q.shape[0]
    o = np.zeros((T, v.shape[1]))
    for t in range(T):
        keys, vals = [], []
        for j in range(M):
            s = [u for u in range(t + 1) if u % M == j]
            keys.append(k[s[-1]] if s else S0k[j])
            vals.append(v[s[-1]] if s else S0v[j])
        sc = scale * np.array([q[t] @ kk for kk in keys])
        p = np.exp(sc - sc.max())
        o[t] = (p / p.sum()) @ np.array(vals)
    return o


def _swa_problem(rng, T=13, M=4, dk=3, dv=2):
    q, k, v, z, _ = _rand(rng, 1, T, 1, dk, dv, M)
    for t in range(T):
        z[0, t, 0, t % M] += 100.0
    g = np.full((1, T, 1), -1e4)                                   # exp(-1e4) == 0: the slot is emptied
    S0k = rng.standard_normal((1, 1, M, dk))
    S0v = rng.standard_normal((1, 1, M, dv))
    return q, k, v, z, g, S0k, S0v


def test_one_hot_router_with_emptying_decay_is_sliding_window_attention():
    rng = np.random.default_rng(501)
    q, k, v, z, g, S0k, S0v = _swa_problem(rng)
    o, Sk, Sv = R.raven_fwd(q, k, v, z, g, 1, S0k, S0v, gate_mode=0, scale=0.8)
    ref = _swa(q[0, :, 0], k[0, :, 0], v[0, :, 0], S0k[0, 0], S0v[0, 0], 4, 0.8)
    assert np.max(np.abs(o[0, :, 0] - ref)) < 1e-12
    T = q.shape[1]
    for j in range(4):                        # the final slots hold the last token of each residue
        s = max(u for u in range(T) if u % 4 == j)
        assert np.array_equal(Sk[0, 0, j], k[0, s, 0]) and np.array_equal(Sv[0, 0, j], v[0, s, 0])


def test_unchosen_slots_are_frozen_bit_for_bit():
    rng = np.random.default_rng(502)
    q, k, v, z, g = _rand(rng, 2, 40, 3, 5, 4, 6)
    z[..., 2] = -50.0                         # never in the top 3
    S0k = rng.standard_normal((2, 3, 6, 5))
    S0v = rng.standard_normal((2, 3, 6, 4))
    _, Sk, Sv = R.raven_fwd(q, k, v, z, g, 3, S0k, S0v)
    assert np.array_equal(Sk[:, :, 2], S0k[:, :, 2]) and np.array_equal(Sv[:, :, 2], S0v[:, :, 2])
    assert not np.allclose(Sk[:, :, 0], S0k[:, :, 0])


def test_dense_equal_router_is_an_exponential_moving_average():
    """K = M with equal logits: r = 1/M on every slot, lam_t = exp(a_t / M), all slots equal (zero
    start), so the softmax is uniform and o_t is the moving average
    sum_s (1 - lam_s) prod_{s < u <= t} lam_u v_s, summed here from its closed form."""
    rng = np.random.default_rng(503)
    T, M = 30, 5
    q, k, v, _, g = _rand(rng, 1, T, 1, 4, 3, M)
    z = np.zeros((1, T, 1, M), dtype=np.float32)
    o, Sk, _ = R.raven_fwd(q, k, v, z, g, M, gate_mode=1, scale=1.3)
    a = -np.log1p(np.exp(g[0, :, 0]))
    lam = np.exp(a / M)
    for t in range(T):
        want = sum((1 - lam[s]) * np.prod(lam[s + 1:t + 1]) * v[0, s, 0] for s in range(t + 1))
        assert np.max(np.abs(o[0, t, 0] - want)) < 1e-12
    want_k = sum((1 - lam[s]) * np.prod(lam[s + 1:]) * k[0, s, 0] for s in range(T))
    assert np.max(np.abs(Sk[0, 0] - want_k[None, :])) < 1e-12


@pytest.mark.parametrize("T,chunk,K,gate_mode", [(150, 64, 3, 1), (70, 16, 1, 0), (33, 64, 8, 1), (64, 8, 2, 1)])
def test_chunk_form_equals_the_token_loop(T, chunk, K, gate_mode):
    rng = np.random.default_rng(510 + T)
    M, dk, dv = 8, 6, 5
    q, k, v, z, g = _rand(rng, 1, T, 1, dk, dv, M)
    if gate_mode == 0:
        g = -np.abs(g) * 2.0
    S0k = rng.standard_normal((1, 1, M, dk))
    S0v = rng.standard_normal((1, 1, M, dv))
    o, Sk, Sv = R.raven_fwd(q, k, v, z, g, K, S0k, S0v, gate_mode=gate_mode, scale=0.7)
    oc, Skc, Svc = R.chunk_form(q[0, :, 0], k[0, :, 0], v[0, :, 0], z[0, :, 0], g[0, :, 0], K, S0k[0, 0], S0v[0, 0],
                                gate_mode=gate_mode, scale=0.7, chunk=chunk)
    assert np.max(np.abs(o[0, :, 0] - oc)) < 1e-11
    assert np.max(np.abs(Sk[0, 0] - Skc)) < 1e-11 and np.max(np.abs(Sv[0, 0] - Svc)) < 1e-11


def _variant(readout_first=False, decay_all=False, unnormalised=False):
    """A copy of the oracle's token step with one plausible mistake planted."""
    def step(Sk, Sv, q, k, v, z, g, K, gate_mode, scale):
        idx, r = R.route(z, K)
        if unnormalised:
            m = 1.0 / (1.0 + np.exp(-np.asarray(z, dtype=np.float64)))
            r = np.where(r > 0, m, 0.0)
        a = R.log_decay(g, gate_mode)[..., None]
        lr = a * np.ones_like(r) / K if decay_all else a * r
        lam, keep = np.exp(lr)[..., None], (-np.expm1(a * r))[..., None]

        def read():
            s = scale * np.einsum("...md,...d->...m", Sk, q)
            p = np.exp(s - np.max(s, axis=-1, keepdims=True))
            return np.einsum("...m,...md->...d", p / p.sum(-1, keepdims=True), Sv)
        o = read() if readout_first else None
        Sk *= lam
        Sk += keep * k[..., None, :]
        Sv *= lam
        Sv += keep * v[..., None, :]
        return read() if o is None else o
    return step


@pytest.mark.parametrize("mistake", ["readout_first", "decay_all", "unnormalised"])
def test_pins_catch_planted_mistakes(monkeypatch, mistake):
    """Each planted mistake fails at least one of the pins above."""
    monkeypatch.setattr(R, "step", _variant(**{mistake: True}))
    failed = 0
    for pin in (test_one_hot_router_with_emptying_decay_is_sliding_window_attention,
                test_unchosen_slots_are_frozen_bit_for_bit, test_dense_equal_router_is_an_exponential_moving_average):
        try:
            pin()
        except AssertionError:
            failed += 1
    assert failed >= 1
