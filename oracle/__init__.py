"""fp64 CPU oracle for the key-axis-gated delta-rule recurrence.

TEST INFRASTRUCTURE ONLY: imported by tests/, by ``__graft_entry__.smoke()`` and
by the CPU-baseline / reference legs of ``bench.py``.  The product path (the CUDA
library and its binding) never imports it.

``gdr_fwd`` and ``gdr_decode_step`` wrap the token-by-token C recurrence in
``gdr_oracle.c`` (the definition written out; see that file's header for the
passages it follows).  ``chunk_wy`` and ``chunk_ut`` restate the chunk-parallel
algebra in fp64 numpy so the tests can check it against the recurrence, as the
"Semidirect Fourier Delta Attention" page reports doing in its results section
(numerical verification against brute force).  ``backward.gdr_bwd`` gives the fp64
reverse-mode gradients of the same recurrence (the oracle of a backward pass).
"""
import ctypes
import os

import numpy as np

from . import build as _build

GATE_LOGDECAY = 0
GATE_NEG_SOFTPLUS = 1

_lib = None


def _load():
    global _lib
    if _lib is None:
        path = _build.build()
        lib = ctypes.CDLL(path)
        dp = ctypes.POINTER(ctypes.c_double)
        lib.oracle_gdr_fwd.argtypes = [ctypes.c_int] * 7 + [ctypes.c_double] + [dp] * 10
        lib.oracle_gdr_fwd.restype = None
        lib.oracle_gdr_decode_step.argtypes = [ctypes.c_int] * 6 + [ctypes.c_double] + [dp] * 9
        lib.oracle_gdr_decode_step.restype = None
        lib.oracle_num_threads.argtypes = []
        lib.oracle_num_threads.restype = ctypes.c_int
        _lib = lib
    return _lib


def _f64(a):
    if a is None:
        return None
    return np.ascontiguousarray(np.asarray(a, dtype=np.float64))


def _ptr(a):
    if a is None:
        return ctypes.POINTER(ctypes.c_double)()
    return a.ctypes.data_as(ctypes.POINTER(ctypes.c_double))


def num_threads() -> int:
    return int(_load().oracle_num_threads())


L2NORM_EPS = 1e-6


def l2_normalise(x):
    """x / sqrt(sum x^2 + 1e-6) over the last axis, in fp64: the L2 normalisation of q and k
    that gated-DeltaNet-family layers (CARVE, KDA) apply before the recurrence,
    with a small epsilon so that a zero vector stays zero."""
    x = np.asarray(x, dtype=np.float64)
    return x / np.sqrt(np.sum(x * x, axis=-1, keepdims=True) + L2NORM_EPS)


def gdr_fwd(q, k, v, g, beta, theta=None, S0=None, gate_mode=GATE_LOGDECAY, scale=1.0,
            want_state=True, w=None, qk_l2norm=False):
    """Token-by-token fp64 forward.

    q, k: [B,T,H,dk]; v: [B,T,H,dv]; g: [B,T,H,dk] (or dk/2 with rotation);
    beta: [B,T,H] erase strength; w: [B,T,H] write strength or None (w = beta);
    theta: [B,T,H,dk/2] or None; S0: [B,H,dv,dk] or None.
    Returns (o [B,T,H,dv], S_T [B,H,dv,dk] or None), both float64.
    """
    q, k, v, g, beta, w, theta, S0 = map(_f64, (q, k, v, g, beta, w, theta, S0))
    if qk_l2norm:
        q, k = l2_normalise(q), l2_normalise(k)
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    rotation = theta is not None
    assert k.shape == q.shape and v.shape == (B, T, H, dv) and beta.shape == (B, T, H)
    assert w is None or w.shape == (B, T, H)
    assert g.shape == (B, T, H, dk // 2 if rotation else dk)
    if rotation:
        assert dk % 2 == 0 and theta.shape == (B, T, H, dk // 2)
    if S0 is not None:
        assert S0.shape == (B, H, dv, dk)
    o = np.zeros((B, T, H, dv))
    S_T = np.zeros((B, H, dv, dk)) if want_state else None
    _load().oracle_gdr_fwd(B, T, H, dk, dv, int(gate_mode), int(rotation), float(scale),
                           _ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(beta), _ptr(w), _ptr(theta),
                           _ptr(S0), _ptr(o), _ptr(S_T))
    return o, S_T


def segment_scan(q, k, v, g, beta, theta=None, S0=None, segment=256, gate_mode=GATE_LOGDECAY, scale=1.0,
                 w=None):
    """The forward in sequence-parallel form, for one head: the affine transfer of the state
    over a stretch of tokens ("Semidirect Fourier Delta Attention" page, *Main contributions*:
    S_end = S_start A + B, exact) applied to segments of the sequence.

    q, k [T,dk]; v [T,dv]; g, beta, w, theta per token as in ``gdr_fwd``; S0 [dv,dk] or None.
    Each segment s (tokens s*segment .. end) is computed independently of the others, twice:
      - from the zero state, giving its outputs o0_t and its write summary B_s = final state;
      - from the identity state (dk x dk) with v = 0, giving o'_t = A_{s,t} (scale q_t) and its
        transfer A_s = final state, with A_{s,t} the product of the segment's token transitions
        D_t (I - beta_t k_t k_t^T) up to t.
    Then a sequential scan over segments gives each start state, S_{s+1} = S_s A_s + B_s, and
    the outputs are o_t = o0_t + S_s o'_t.  Returns (o [T,dv], S_T [dv,dk]).
    """
    q, k, v, g, beta, theta, S0, w = map(_f64, (q, k, v, g, beta, theta, S0, w))
    T, dk = q.shape
    dv = v.shape[1]
    one = lambda a, t0, t1: None if a is None else a[None, t0:t1, None]
    S = np.zeros((dv, dk)) if S0 is None else S0.copy()
    o = np.zeros((T, dv))
    for t0 in range(0, T, segment):
        t1 = min(t0 + segment, T)
        args = (one(q, t0, t1), one(k, t0, t1))
        rest = (one(g, t0, t1), one(beta, t0, t1), one(theta, t0, t1))
        o0, B_s = gdr_fwd(*args, one(v, t0, t1), *rest, None, gate_mode=gate_mode, scale=scale,
                          w=one(w, t0, t1))
        oI, A_s = gdr_fwd(*args, np.zeros((1, t1 - t0, 1, dk)), *rest, np.eye(dk)[None, None],
                          gate_mode=gate_mode, scale=scale, w=one(w, t0, t1))
        o[t0:t1] = o0[0, :, 0] + oI[0, :, 0] @ S.T
        S = S @ A_s[0, 0] + B_s[0, 0]
    return o, S


def chunk_means(o, chunk=64):
    """Mean of the outputs over each chunk ("CARVE" page, section 2.1: the chunk mean
    m_c = (1/L) sum of o_t over chunk c, the content signal of its content-aware erase).

    o: [B,T,H,dv].  Chunk c holds tokens c*chunk .. min((c+1)*chunk, T) - 1 and L is the
    number of those tokens, so a short last chunk is averaged over its own tokens.
    Returns [B, ceil(T/chunk), H, dv] float64.
    """
    o = np.asarray(o, dtype=np.float64)
    B, T, H, dv = o.shape
    nc = (T + chunk - 1) // chunk
    m = np.zeros((B, nc, H, dv))
    for c in range(nc):
        t0, t1 = c * chunk, min((c + 1) * chunk, T)
        m[:, c] = o[:, t0:t1].sum(axis=1) / (t1 - t0)
    return m


def gdr_decode_step(q, k, v, g, beta, S, theta=None, gate_mode=GATE_LOGDECAY, scale=1.0, w=None,
                    qk_l2norm=False):
    """One fp64 decode step (w: write strength [N,H] or None for w = beta).
    S [N,H,dv,dk] is NOT modified; returns (o, S_new)."""
    q, k, v, g, beta, w, theta = map(_f64, (q, k, v, g, beta, w, theta))
    if qk_l2norm:
        q, k = l2_normalise(q), l2_normalise(k)
    S_new = np.array(S, dtype=np.float64, copy=True, order="C")
    N, H, dk = q.shape
    dv = v.shape[-1]
    rotation = theta is not None
    assert g.shape == (N, H, dk // 2 if rotation else dk) and beta.shape == (N, H)
    o = np.zeros((N, H, dv))
    _load().oracle_gdr_decode_step(N, H, dk, dv, int(gate_mode), int(rotation), float(scale),
                                   _ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(beta), _ptr(w),
                                   _ptr(theta), _ptr(S_new), _ptr(o))
    return o, S_new
