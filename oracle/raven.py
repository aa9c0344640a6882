"""fp64 oracle of Raven's routed slot memory (a second workload of the recurrence family).

TEST INFRASTRUCTURE ONLY, like the rest of ``oracle/``: imported by tests/, by
``__graft_entry__.smoke()`` and by the CPU legs of ``bench.py``; never by the product path.

Source: the page "Raven: High-Recall Sequence Modeling with Sparse Memory Routing", sections
2.1 (routing slot memories: M slots, a router r_t in R^M deciding which slots are written and
decayed) and 2.2 (Raven: separate key and value slot states; router scores m_t = sigmoid of a
projection of x_t, the top K kept and the rest set to zero, the kept ones normalised; decay only
on the chosen slots, S_t = exp(a_t r_t) * S_{t-1} + (1 - exp(a_t r_t)) * k_t^T, so an unchosen
slot, r = 0, is frozen; no short convolution).  Readings (the page leaves these open):
  - the router's logits z_t = W x_t are an input (the projection is the layer's, like q, k, v);
  - the top K are taken on the logits (the sigmoid is monotone), ties to the lower slot index;
    the kept scores are normalised to sum to one, r_t[i] = m_t[i] / sum_{j in top K} m_t[j];
  - a_t is one log-decay per token and head: a_t = g_t (gate mode 0) or -softplus(g_t) (mode 1);
  - the value state follows the same rule with v_t in place of k_t;
  - the readout is softmax attention over the M slots of the updated state,
    o_t = sum_i softmax_i(scale q_t . S^k_t[i]) S^v_t[i]; with a one-hot router cycling through
    the slots and a decay that empties the chosen slot this is exactly sliding-window attention
    over the last M tokens, the special case section 2.1 names.

``raven_fwd`` is the definition written out token by token; ``chunk_form`` restates it chunk by
chunk (per-slot cumulative log-decays, the state's part of the scores and outputs, and the
chunk's own writes as sums over the tokens that chose each slot), the form a chunked kernel
takes; the tests hold it to the token loop.
"""
import numpy as np


def route(z, K):
    """Top-K routing of logits z [..., M]: returns (idx [..., K], r [..., M]) with idx the chosen
    slots in decreasing logit order (ties: lower index first) and r the normalised weights of the
    chosen slots (zero elsewhere)."""
    z = np.asarray(z, dtype=np.float64)
    idx = np.argsort(-z, axis=-1, kind="stable")[..., :K]
    m = 1.0 / (1.0 + np.exp(-np.take_along_axis(z, idx, axis=-1)))
    r = np.zeros_like(z)
    np.put_along_axis(r, idx, m / np.sum(m, axis=-1, keepdims=True), axis=-1)
    return idx, r


def log_decay(g, gate_mode):
    """a_t from the gate input: g itself (mode 0) or -softplus(g) (mode 1)."""
    g = np.asarray(g, dtype=np.float64)
    if gate_mode == 1:
        return -(np.maximum(g, 0.0) + np.log1p(np.exp(-np.abs(g))))
    return g


def step(Sk, Sv, q, k, v, z, g, K, gate_mode, scale):
    """One token for every (batch, head) at once: Sk, Sv [..., M, d] updated in place; q, k [..., dk],
    v [..., dv], z [..., M], g [...].  Returns o [..., dv]."""
    _, r = route(z, K)
    lr = log_decay(g, gate_mode)[..., None] * r            # a_t r_t (zero on unchosen slots)
    lam = np.exp(lr)[..., None]
    keep = -np.expm1(lr)[..., None]                        # 1 - exp(a_t r_t)
    Sk *= lam
    Sk += keep * k[..., None, :]
    Sv *= lam
    Sv += keep * v[..., None, :]
    s = scale * np.einsum("...md,...d->...m", Sk, q)
    p = np.exp(s - np.max(s, axis=-1, keepdims=True))
    p /= np.sum(p, axis=-1, keepdims=True)
    return np.einsum("...m,...md->...d", p, Sv)


def raven_fwd(q, k, v, z, g, K, S0k=None, S0v=None, gate_mode=1, scale=1.0):
    """Token loop over [B,T,H,*] inputs: q, k [B,T,H,dk]; v [B,T,H,dv]; z [B,T,H,M] router
    logits; g [B,T,H] decay gate; S0k [B,H,M,dk], S0v [B,H,M,dv] or None (zero).
    Returns (o [B,T,H,dv], Sk_T, Sv_T)."""
    f = lambda a: None if a is None else np.asarray(a, dtype=np.float64)
    q, k, v, z, g, S0k, S0v = map(f, (q, k, v, z, g, S0k, S0v))
    B, T, H, dk = q.shape
    dv, M = v.shape[-1], z.shape[-1]
    Sk = np.zeros((B, H, M, dk)) if S0k is None else S0k.copy()
    Sv = np.zeros((B, H, M, dv)) if S0v is None else S0v.copy()
    o = np.zeros((B, T, H, dv))
    for t in range(T):
        o[:, t] = step(Sk, Sv, q[:, t], k[:, t], v[:, t], z[:, t], g[:, t], K, gate_mode, scale)
    return o, Sk, Sv


def chunk_form(q, k, v, z, g, K, S0k=None, S0v=None, gate_mode=1, scale=1.0, chunk=64):
    """The same forward for one head (q, k [T,dk], v [T,dv], z [T,M], g [T]) chunk by chunk.
    Per chunk with start states Sk0, Sv0 and lam_t[i] = sum over the chunk's tokens u <= t of
    a_u r_u[i] (the slot's cumulative log-decay):
        scores[t,i] = scale e^{lam_t[i]} q_t . Sk0[i]
                      + scale sum_{s <= t, i chosen at s} (q_t . k_s) c_s[i] e^{lam_t[i] - lam_s[i]}
        p_t = softmax(scores[t])
        o_t = sum_i p_t[i] e^{lam_t[i]} Sv0[i] + sum_{s <= t} w[t,s] v_s,
              w[t,s] = sum_{i chosen at s} p_t[i] c_s[i] e^{lam_t[i] - lam_s[i]}
        Sk_L[i] = e^{lam_L[i]} Sk0[i] + sum_{s: i chosen at s} c_s[i] e^{lam_L[i] - lam_s[i]} k_s
    (likewise Sv_L), with c_s[i] = 1 - e^{a_s r_s[i]}.  Every exponent is <= 0."""
    q, k, v, z = (np.asarray(a, dtype=np.float64) for a in (q, k, v, z))
    T, dk = q.shape
    dv, M = v.shape[1], z.shape[1]
    Sk = np.zeros((M, dk)) if S0k is None else np.array(S0k, dtype=np.float64)
    Sv = np.zeros((M, dv)) if S0v is None else np.array(S0v, dtype=np.float64)
    idx, r = route(z, K)
    lr = log_decay(g, gate_mode)[:, None] * r                 # [T, M]
    c = -np.expm1(lr)
    o = np.zeros((T, dv))
    for t0 in range(0, T, chunk):
        t1 = min(t0 + chunk, T)
        L = t1 - t0
        lam = np.cumsum(lr[t0:t1], axis=0)                     # [L, M]
        A = scale * (q[t0:t1] @ k[t0:t1].T)                    # [L, L]
        sc = scale * np.exp(lam) * (q[t0:t1] @ Sk.T)
        for t in range(L):
            for s in range(t + 1):
                for i in idx[t0 + s]:
                    sc[t, i] += A[t, s] * c[t0 + s, i] * np.exp(lam[t, i] - lam[s, i])
        p = np.exp(sc - np.max(sc, axis=1, keepdims=True))
        p /= np.sum(p, axis=1, keepdims=True)
        w = np.zeros((L, L))
        for t in range(L):
            for s in range(t + 1):
                for i in idx[t0 + s]:
                    w[t, s] += p[t, i] * c[t0 + s, i] * np.exp(lam[t, i] - lam[s, i])
        o[t0:t1] = (p * np.exp(lam)) @ Sv + w @ v[t0:t1]
        Sk_new = np.exp(lam[-1])[:, None] * Sk
        Sv_new = np.exp(lam[-1])[:, None] * Sv
        for s in range(L):
            for i in idx[t0 + s]:
                f = c[t0 + s, i] * np.exp(lam[-1, i] - lam[s, i])
                Sk_new[i] += f * k[t0 + s]
                Sv_new[i] += f * v[t0 + s]
        Sk, Sv = Sk_new, Sv_new
    return o, Sk, Sv
