"""Seeded synthetic inputs for the gated delta-rule workloads.

This module only draws random numbers and lays them out; it holds none of the
recurrence's arithmetic.  Tests, the bench and the smoke check take their inputs
from here and hand the very same bytes to the CUDA library and to the CPU oracle.

Random numbers come from a counter-based SplitMix64 stream (Steele, Lea and
Flood, "Fast splittable pseudorandom number generators", OOPSLA 2014): the i-th
64-bit word of a stream with key s is mix(s + (i+1) * 0x9E3779B97F4A7C15).
Uniforms take the top 53 bits; normals use the Box-Muller transform (cosine
branch only).  Every tensor draws from its own stream, keyed by the seed and the
tensor's name, so the values do not depend on the order of generation.

The workload recipe (from the configurations the benchmark is quoted on):
q and k are N(0,1) and L2-normalised per token in fp32, then rounded to bf16
(round to nearest even) when the run is in bf16 mode; v is N(0,1); the raw gate a
is N(0,1) and the kernels apply g = -softplus(a) themselves; beta = sigmoid(N(0,1)).
"""
from __future__ import annotations

import os
import zlib
from concurrent.futures import ThreadPoolExecutor
from dataclasses import dataclass
from typing import Optional

import numpy as np

_GAMMA = np.uint64(0x9E3779B97F4A7C15)
_M1 = np.uint64(0xBF58476D1CE4E5B9)
_M2 = np.uint64(0x94D049BB133111EB)

GATE_LOGDECAY = 0
GATE_NEG_SOFTPLUS = 1


def _mix(z: np.ndarray) -> np.ndarray:
    z = (z ^ (z >> np.uint64(30))) * _M1
    z = (z ^ (z >> np.uint64(27))) * _M2
    return z ^ (z >> np.uint64(31))


def _stream_key(seed: int, name: str) -> np.uint64:
    with np.errstate(over="ignore"):
        s = _mix(np.array([np.uint64(seed & 0xFFFFFFFFFFFFFFFF)], dtype=np.uint64))[0]
        s = s ^ np.uint64(zlib.crc32(name.encode()))
        return _mix(np.array([s], dtype=np.uint64))[0]


def uniform(seed: int, name: str, n: int, offset: int = 0) -> np.ndarray:
    """n uniforms in [0, 1) (float64) from stream (seed, name), words offset.. offset+n-1."""
    key = _stream_key(seed, name)
    out = np.empty(n, dtype=np.float64)
    block = 1 << 22
    with np.errstate(over="ignore"):
        for b0 in range(0, n, block):
            m = min(block, n - b0)
            idx = np.arange(offset + b0 + 1, offset + b0 + 1 + m, dtype=np.uint64)
            z = _mix(key + idx * _GAMMA)
            out[b0:b0 + m] = (z >> np.uint64(11)).astype(np.float64) * (1.0 / 9007199254740992.0)
    return out


def _normal_block(seed, name, b0, m):
    u = uniform(seed, name, 2 * m, offset=2 * b0)
    u1 = 1.0 - u[0::2]                      # (0, 1]
    u2 = u[1::2]
    return np.sqrt(-2.0 * np.log(u1)) * np.cos(2.0 * np.pi * u2)


_POOL = None


def _pool():
    global _POOL
    if _POOL is None:
        _POOL = ThreadPoolExecutor(max_workers=max(1, min(16, os.cpu_count() or 1)))
    return _POOL


def normal(seed: int, name: str, shape, mean: float = 0.0, std: float = 1.0) -> np.ndarray:
    """Normals (float64) of the given shape from stream (seed, name)."""
    n = int(np.prod(shape))
    out = np.empty(n, dtype=np.float64)
    block = 1 << 21
    starts = list(range(0, n, block))

    def work(b0):
        m = min(block, n - b0)
        out[b0:b0 + m] = _normal_block(seed, name, b0, m)

    if len(starts) > 1:
        list(_pool().map(work, starts))
    else:
        for b0 in starts:
            work(b0)
    return (mean + std * out).reshape(shape)


def to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """float32 -> bf16 bit pattern (uint16), round to nearest even."""
    b = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32)
    bias = ((b >> np.uint32(16)) & np.uint32(1)) + np.uint32(0x7FFF)
    return ((b + bias) >> np.uint32(16)).astype(np.uint16)


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    return (np.ascontiguousarray(b, dtype=np.uint16).astype(np.uint32) << np.uint32(16)).view(np.float32)


def _l2_normalise_rows(x: np.ndarray) -> np.ndarray:
    x32 = x.astype(np.float32)
    nrm = np.sqrt(np.sum(x32 * x32, axis=-1, keepdims=True, dtype=np.float32))
    return (x32 / np.maximum(nrm, np.float32(1e-12))).astype(np.float32)


@dataclass
class FwdInputs:
    """One forward problem.  Arrays are host numpy; bf16 tensors are uint16 bit patterns."""
    B: int
    T: int
    H: int
    dk: int
    dv: int
    chunk: int
    dtype: str                  # "bf16" or "f32": storage of q, k, v and o
    gate_mode: int
    rotation: bool
    q: np.ndarray
    k: np.ndarray
    v: np.ndarray
    g: np.ndarray               # float32 [B,T,H,dk] or [B,T,H,dk/2]
    beta: np.ndarray            # float32 [B,T,H]
    theta: Optional[np.ndarray] = None   # float32 [B,T,H,dk/2]
    S0: Optional[np.ndarray] = None      # float32 [B,H,dv,dk]
    scale: float = 1.0
    name: str = ""

    def widened(self, key: str) -> Optional[np.ndarray]:
        """The exact fp64 value of an input array (bf16 widened bit-exactly)."""
        a = getattr(self, key)
        if a is None:
            return None
        if a.dtype == np.uint16:
            return bf16_bits_to_f32(a).astype(np.float64)
        return a.astype(np.float64)

    def head_slice(self, b: int, h: int) -> "FwdInputs":
        """The same problem restricted to one (batch, head) pair."""
        def sl(a):
            return None if a is None else np.ascontiguousarray(a[b:b + 1, :, h:h + 1])
        return FwdInputs(1, self.T, 1, self.dk, self.dv, self.chunk, self.dtype, self.gate_mode,
                         self.rotation, sl(self.q), sl(self.k), sl(self.v), sl(self.g),
                         sl(self.beta), sl(self.theta),
                         None if self.S0 is None else np.ascontiguousarray(self.S0[b:b + 1, h:h + 1]),
                         self.scale, self.name)

    @property
    def nbytes_algorithmic(self) -> int:
        """Bytes the method must move: inputs read once, o and S_T written once."""
        s = 2 if self.dtype == "bf16" else 4
        tok = self.B * self.T * self.H
        n = tok * (2 * self.dk * s + self.dv * s + self.g.shape[-1] * 4 + 4 + self.dv * s)
        if self.theta is not None:
            n += tok * self.theta.shape[-1] * 4
        n += self.B * self.H * self.dv * self.dk * 4           # S_T written
        if self.S0 is not None:
            n += self.B * self.H * self.dv * self.dk * 4       # S0 read
        return n


def make_fwd(B, T, H, dk, dv, chunk=64, dtype="bf16", seed=0, rotation=False,
             gate="normal", s0_std: Optional[float] = None, scale=1.0, name="") -> FwdInputs:
    """Random forward problem following the workloads' recipe.

    gate: "normal"  -> raw gate a ~ N(0,1), kernels apply g = -softplus(a);
          "slow"    -> a = -x with x ~ N(2,1), so g = -softplus(-x) = log sigmoid(x);
    s0_std: None for a zero initial state (S0 omitted), else S0 ~ N(0, s0_std^2).
    """
    q = _l2_normalise_rows(normal(seed, "q", (B, T, H, dk)))
    k = _l2_normalise_rows(normal(seed, "k", (B, T, H, dk)))
    v = normal(seed, "v", (B, T, H, dv)).astype(np.float32)
    ng = dk // 2 if rotation else dk
    if gate == "slow":
        a = -normal(seed, "a", (B, T, H, ng), mean=2.0, std=1.0)
    else:
        a = normal(seed, "a", (B, T, H, ng))
    beta = 1.0 / (1.0 + np.exp(-normal(seed, "beta", (B, T, H))))
    theta = None
    if rotation:
        theta = (uniform(seed, "theta", B * T * H * (dk // 2)) * 2.0 - 1.0) * np.pi
        theta = theta.reshape(B, T, H, dk // 2).astype(np.float32)
    S0 = None
    if s0_std is not None:
        S0 = normal(seed, "S0", (B, H, dv, dk), std=s0_std).astype(np.float32)
    if dtype == "bf16":
        q, k, v = to_bf16_bits(q), to_bf16_bits(k), to_bf16_bits(v)
    elif dtype != "f32":
        raise ValueError(dtype)
    return FwdInputs(B, T, H, dk, dv, chunk, dtype, GATE_NEG_SOFTPLUS, rotation, q, k, v,
                     a.astype(np.float32), beta.astype(np.float32), theta, S0, scale, name)


# The five workloads: tiny fp32 parity case, the headline bf16 shape, the
# 1.3B-layer training shape with a slow decay and a random initial state, the
# block-rotation variant, and recurrent decode.
FWD_CONFIGS = {
    "tiny_f32": dict(B=1, H=2, T=256, dk=32, dv=32, chunk=64, dtype="f32", seed=0),
    "b4_h16_t4096_d128": dict(B=4, H=16, T=4096, dk=128, dv=128, chunk=64, dtype="bf16", seed=1),
    "b16_h12_t4096_d128_slow_s0": dict(B=16, H=12, T=4096, dk=128, dv=128, chunk=64, dtype="bf16",
                                       seed=2, gate="slow", s0_std=0.02),
    "b2_h16_t8192_d128_rot": dict(B=2, H=16, T=8192, dk=128, dv=128, chunk=64, dtype="bf16",
                                  seed=3, rotation=True),
}

DECODE_CONFIG = dict(N=256, H=16, dk=128, dv=128, steps=1000, dtype="bf16", seed=4, s_std=0.02)


def make_config(name: str, **overrides) -> FwdInputs:
    kw = dict(FWD_CONFIGS[name])
    kw.update(overrides)
    return make_fwd(name=name, **kw)


@dataclass
class DecodeInputs:
    N: int
    H: int
    dk: int
    dv: int
    dtype: str
    gate_mode: int
    rotation: bool
    q: np.ndarray               # [steps, N, H, dk]
    k: np.ndarray
    v: np.ndarray               # [steps, N, H, dv]
    g: np.ndarray               # [steps, N, H, dk or dk/2] float32
    beta: np.ndarray            # [steps, N, H] float32
    theta: Optional[np.ndarray] = None
    S: Optional[np.ndarray] = None       # [N, H, dv, dk] float32 initial state
    scale: float = 1.0

    def widened(self, key: str, step: Optional[int] = None):
        a = getattr(self, key)
        if a is None:
            return None
        if step is not None and key != "S":
            a = a[step]
        if a.dtype == np.uint16:
            return bf16_bits_to_f32(a).astype(np.float64)
        return a.astype(np.float64)


def make_write_strength(seed, shape) -> np.ndarray:
    """A write strength w = sigmoid(N(0,1)) separate from beta (fp32), for the untied rule."""
    return (1.0 / (1.0 + np.exp(-normal(seed, "w", shape)))).astype(np.float32)


def make_decode(N, H, dk, dv, steps, dtype="bf16", seed=4, s_std=0.02, rotation=False,
                scale=1.0) -> DecodeInputs:
    """Per-step single-token inputs for N independent sequences, plus the state S."""
    q = _l2_normalise_rows(normal(seed, "dq", (steps, N, H, dk)))
    k = _l2_normalise_rows(normal(seed, "dk", (steps, N, H, dk)))
    v = normal(seed, "dv", (steps, N, H, dv)).astype(np.float32)
    ng = dk // 2 if rotation else dk
    a = normal(seed, "da", (steps, N, H, ng)).astype(np.float32)
    beta = (1.0 / (1.0 + np.exp(-normal(seed, "dbeta", (steps, N, H))))).astype(np.float32)
    theta = None
    if rotation:
        theta = ((uniform(seed, "dtheta", steps * N * H * (dk // 2)) * 2.0 - 1.0) * np.pi)
        theta = theta.reshape(steps, N, H, dk // 2).astype(np.float32)
    S = normal(seed, "dS", (N, H, dv, dk), std=s_std).astype(np.float32)
    if dtype == "bf16":
        q, k, v = to_bf16_bits(q), to_bf16_bits(k), to_bf16_bits(v)
    return DecodeInputs(N, H, dk, dv, dtype, GATE_NEG_SOFTPLUS, rotation, q, k, v, a, beta,
                        theta, S, scale)


@dataclass
class RavenInputs:
    """One problem of Raven's routed slot memory (arrays host numpy, q / k / v bf16 bit patterns)."""
    B: int
    T: int
    H: int
    d: int
    K: int
    gate_mode: int
    q: np.ndarray               # [B,T,H,d] bf16 bits
    k: np.ndarray
    v: np.ndarray
    z: np.ndarray               # [B,T,H,M] float32 router logits
    g: np.ndarray               # [B,T,H] float32 decay gate
    S0k: Optional[np.ndarray]   # [B,H,M,d] float32 or None
    S0v: Optional[np.ndarray]
    scale: float
    name: str = ""

    def widened(self, key: str) -> Optional[np.ndarray]:
        a = getattr(self, key)
        if a is None:
            return None
        if a.dtype == np.uint16:
            return bf16_bits_to_f32(a).astype(np.float64)
        return a.astype(np.float64)


def make_raven(B, T, H, d, K=8, seed=5, gate_mode=GATE_NEG_SOFTPLUS, s0_std: Optional[float] = None, M=64,
               scale: Optional[float] = None, name="") -> RavenInputs:
    """Random Raven problem: q, k, v ~ N(0,1) rounded to bf16, router logits z ~ N(0,1) per slot,
    the gate ~ N(0,1) (a raw gate for GATE_NEG_SOFTPLUS) or -|N(0,1)| (a log-decay for
    GATE_LOGDECAY), start states N(0, s0_std^2) or none, scale 1/sqrt(d) unless given."""
    q = to_bf16_bits(normal(seed, "rq", (B, T, H, d)))
    k = to_bf16_bits(normal(seed, "rk", (B, T, H, d)))
    v = to_bf16_bits(normal(seed, "rv", (B, T, H, d)))
    z = normal(seed, "rz", (B, T, H, M)).astype(np.float32)
    g = normal(seed, "rg", (B, T, H))
    g = (g if gate_mode == GATE_NEG_SOFTPLUS else -np.abs(g)).astype(np.float32)
    S0k = S0v = None
    if s0_std is not None:
        S0k = normal(seed, "rS0k", (B, H, M, d), std=s0_std).astype(np.float32)
        S0v = normal(seed, "rS0v", (B, H, M, d), std=s0_std).astype(np.float32)
    return RavenInputs(B, T, H, d, K, gate_mode, q, k, v, z, g, S0k, S0v,
                       float(d ** -0.5 if scale is None else scale), name)


# Raven's workload: the headline forward's shape (B=4, H=16, T=4096, d=128) with 64 slots and
# top-8 routing (the page fixes neither number).
RAVEN_CONFIGS = {
    "raven_b4_h16_t4096_d128": dict(B=4, T=4096, H=16, d=128, K=8, seed=5),
}


def make_raven_config(name: str, **overrides) -> RavenInputs:
    kw = dict(RAVEN_CONFIGS[name])
    kw.update(overrides)
    return make_raven(name=name, **kw)
